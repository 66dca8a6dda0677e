// Plain fp64 CPU oracle for importance-sampled block-sparse attention.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and
// the benchmark's CPU-baseline leg may load this library.  It shares no code,
// header or constant table with the CUDA path under block_sparse_importance_b200/.
//
// What it restates (all page citations are to the titles below):
//   [AB]  "AB-Attention: Accurate Block Attention for Accelerating Video
//         Diffusion Transformers" (abstract and the podcast discussion of the
//         method: IBCS, SIP, logit shifts, fine-grained tiled execution).
//   [IG]  "InstaGen: Group-Shared Importance Sampling for Fast Video
//         Generation" (abstract: exact set + inverse-probability-weighted sample,
//         one sample per query cluster).
//   [PH]  Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
//         1, 2, 3" (SC'11): the Philox4x64-10 counter-based generator.
//   [IC]  "iCATS: Fast Video Generation via Interaction-Aware Sparse Attention
//         and Timestep-Adaptive Sparsity" (AI summary, "Approach": top-p and
//         the merging of query-cluster tails).
//
// The pages give no equations; every rule marked (reading) below is the
// plainest reading that the rest of the pages supports.
//
// Parity pins (tests/test_oracle_*.py): Philox vs numpy's Philox and the
// generator's published known-answer vectors; top-k vs brute-force sort;
// k-means fixed-point invariants; mass sum invariant and the one-cluster
// closed form; capping (sum of pi = n_s, pi <= 1, minimality); exact
// inclusion probabilities and exact unbiasedness of the weighted numerator
// and denominator by integration over the uniform; the pages' worked example
// (pi = 1/4 counts four times); the dense limit against a library attention.
// Token clustering (the permuted layout): brute-force nearest centroid, the
// stable sort against a library stable argsort, the mean update against
// numpy, the one-cluster closed form, a non-increasing objective, and the
// recovery of well-separated generated clusters.  Tail merging: worked
// examples done by hand (join order, Hamming-nearest choice, ties), the closed
// forms for identical and disjoint plans, and the schedule's rules on random
// inputs (partition of the tails, slots, unions, no merge that costs work).
// Choices the pages leave open (each is a stated reading; the functions that
// make them are pinned by the checks above, but no page value can pin the
// choice itself, so the GPU matches the oracle on them by construction): the
// k-means initialisation, the ln(L_b) term of the mass, tie-breaks, canonical
// plan order, the 2^31 weight quantisation, the clustering's round count.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <iterator>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

double bf16_value(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

uint32_t float_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

float bits_float(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

typedef unsigned __int128 u128;

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// [PH] Philox4x64-10: ten rounds of the 4x64 Philox S-box (two 64x64->128
// multiplications with the paper's multipliers, xor with the round key),
// the key bumped by the two Weyl constants between rounds.
// ---------------------------------------------------------------------------
void ref_philox4x64_10(const uint64_t* ctr, const uint64_t* key, uint64_t* out) {
  const uint64_t M0 = 0xD2E7470EE14C6C93ULL, M1 = 0xCA5A826395121157ULL;
  const uint64_t W0 = 0x9E3779B97F4A7C15ULL, W1 = 0xBB67AE8584CAA73BULL;
  uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint64_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += W0;
      k1 += W1;
    }
    u128 p0 = static_cast<u128>(M0) * c0;
    u128 p1 = static_cast<u128>(M1) * c2;
    uint64_t hi0 = static_cast<uint64_t>(p0 >> 64), lo0 = static_cast<uint64_t>(p0);
    uint64_t hi1 = static_cast<uint64_t>(p1 >> 64), lo1 = static_cast<uint64_t>(p1);
    uint64_t n0 = hi1 ^ c1 ^ k0;
    uint64_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

// The one uniform a query group draws (reading): key = (seed, 0), counter =
// (group, head, batch, 0); U = high 32 bits of output word 0; u = U * 2^-32.
uint32_t ref_group_uniform(uint64_t seed, int32_t batch, int32_t head, int32_t group) {
  uint64_t ctr[4] = {static_cast<uint64_t>(static_cast<uint32_t>(group)),
                     static_cast<uint64_t>(static_cast<uint32_t>(head)),
                     static_cast<uint64_t>(static_cast<uint32_t>(batch)), 0};
  uint64_t key[2] = {seed, 0};
  uint64_t out[4];
  ref_philox4x64_10(ctr, key, out);
  return static_cast<uint32_t>(out[0] >> 32);
}

// ---------------------------------------------------------------------------
// [AB] IBCS, key side: "representatives score small key blocks"; key blocks
// are summarised by their means.  Block b holds rows [b*Bk, min((b+1)*Bk, N));
// L_b is its row count (the tail block keeps only its valid rows, reading).
// k: one head, [N, d] bf16 bits.  kbar: [nK, d].  L: [nK].
// ---------------------------------------------------------------------------
void ref_key_means(const uint16_t* k, int32_t N, int32_t d, int32_t Bk, double* kbar, int32_t* L) {
  const int32_t nK = (N + Bk - 1) / Bk;
  for (int32_t b = 0; b < nK; ++b) {
    const int32_t r0 = b * Bk, r1 = std::min(N, r0 + Bk);
    L[b] = r1 - r0;
    for (int32_t j = 0; j < d; ++j) {
      double s = 0.0;
      for (int32_t r = r0; r < r1; ++r) s += bf16_value(k[static_cast<int64_t>(r) * d + j]);
      kbar[static_cast<int64_t>(b) * d + j] = s / (r1 - r0);
    }
  }
}

// ---------------------------------------------------------------------------
// [AB] IBCS, query side: queries are clustered only within their own query
// block; each cluster yields a representative and a weight equal to its size.
// Lloyd's k-means (reading):
//   init  mu_c = q[floor(c * n / C)], c = 0..C-1 (evenly spaced rows);
//   iterate `iters` times: assign every row to argmin_c ||q - mu_c||^2 (ties to
//   the lower c), then move every non-empty cluster's mu_c to the mean of its
//   rows (an empty cluster keeps its mu_c);
//   counts are the sizes of the last assignment.
// q: [n, d] bf16 bits of the group's rows.  mu: [C, d].  counts: [C].
// iters >= 1 (the callers check it).
// Returns 1 when some assignment was decided by a margin smaller than
// tie_rel * (||q||^2 + ||mu||^2): such a group's clustering is not unique at
// single precision, so a single-precision implementation may legitimately
// differ from this one there.
// ---------------------------------------------------------------------------
int32_t ref_kmeans_group(const uint16_t* q, int32_t n, int32_t d, int32_t C, int32_t iters,
                         double tie_rel, double* mu, int32_t* counts) {
  std::vector<double> x(static_cast<size_t>(n) * d);
  for (int64_t i = 0; i < static_cast<int64_t>(n) * d; ++i) x[i] = bf16_value(q[i]);
  for (int32_t c = 0; c < C; ++c) {
    const int64_t r = (static_cast<int64_t>(c) * n) / C;
    for (int32_t j = 0; j < d; ++j) mu[static_cast<int64_t>(c) * d + j] = x[r * d + j];
  }
  std::vector<int32_t> assign(n, 0);
  std::vector<double> sum(static_cast<size_t>(C) * d);
  int32_t ambiguous = 0;
  for (int32_t c = 0; c < C; ++c) counts[c] = 0;
  for (int32_t it = 0; it < iters; ++it) {
    for (int32_t r = 0; r < n; ++r) {
      double best = INFINITY, second = INFINITY, qq = 0.0, mm_best = 0.0, mm_second = 0.0;
      int32_t arg = 0;
      for (int32_t j = 0; j < d; ++j) qq += x[static_cast<int64_t>(r) * d + j] * x[static_cast<int64_t>(r) * d + j];
      for (int32_t c = 0; c < C; ++c) {
        double dist = 0.0, mm = 0.0;
        for (int32_t j = 0; j < d; ++j) {
          const double m = mu[static_cast<int64_t>(c) * d + j];
          const double t = x[static_cast<int64_t>(r) * d + j] - m;
          dist += t * t;
          mm += m * m;
        }
        if (dist < best) {
          second = best;
          mm_second = mm_best;
          best = dist;
          mm_best = mm;
          arg = c;
        } else if (dist < second) {
          second = dist;
          mm_second = mm;
        }
      }
      if (C > 1 && second - best <= tie_rel * (qq + std::max(mm_best, mm_second))) ambiguous = 1;
      assign[r] = arg;
    }
    std::fill(sum.begin(), sum.end(), 0.0);
    for (int32_t c = 0; c < C; ++c) counts[c] = 0;
    for (int32_t r = 0; r < n; ++r) {
      counts[assign[r]] += 1;
      for (int32_t j = 0; j < d; ++j) sum[static_cast<int64_t>(assign[r]) * d + j] += x[static_cast<int64_t>(r) * d + j];
    }
    for (int32_t c = 0; c < C; ++c) {
      if (counts[c] == 0) continue;
      for (int32_t j = 0; j < d; ++j) mu[static_cast<int64_t>(c) * d + j] = sum[static_cast<int64_t>(c) * d + j] / counts[c];
    }
  }
  return ambiguous;
}

// ---------------------------------------------------------------------------
// [AB] estimated attention mass of one query group over all key blocks.
// A block of L_b keys near its mean kbar_b carries about L_b * exp(scale *
// mu_c . kbar_b) of cluster c's unnormalised attention, so (reading)
//   l_{c,b} = scale * mu_c . kbar_b + ln L_b,
//   p_{c,b} = softmax over b of l_{c,b},
//   m_b     = sum_c n_c * p_{c,b}        (cluster-size weighted),
// and sum_b m_b = n (the group's row count) is the expected attention mass
// the group's queries put on the whole sequence.
// ---------------------------------------------------------------------------
void ref_mass_group(const double* mu, const int32_t* counts, int32_t C, const double* kbar,
                    const int32_t* L, int32_t nK, int32_t d, double scale, double* mass) {
  std::vector<double> l(nK);
  for (int32_t b = 0; b < nK; ++b) mass[b] = 0.0;
  for (int32_t c = 0; c < C; ++c) {
    if (counts[c] == 0) continue;
    double mx = -INFINITY;
    for (int32_t b = 0; b < nK; ++b) {
      double dot = 0.0;
      for (int32_t j = 0; j < d; ++j) dot += mu[static_cast<int64_t>(c) * d + j] * kbar[static_cast<int64_t>(b) * d + j];
      l[b] = scale * dot + std::log(static_cast<double>(L[b]));
      mx = std::max(mx, l[b]);
    }
    double z = 0.0;
    for (int32_t b = 0; b < nK; ++b) z += std::exp(l[b] - mx);
    for (int32_t b = 0; b < nK; ++b) mass[b] += counts[c] * (std::exp(l[b] - mx) / z);
  }
}

// Whole scorer over [B, H, N, d].  Groups are rows [off[g], off[g+1]) (the
// same for every batch and head).  mass: [B, H, G, nK]; centroids
// [B, H, G, C, d]; counts [B, H, G, C]; ambiguous [B, H, G] (may be NULL).
void ref_score(const uint16_t* q, const uint16_t* k, int32_t B, int32_t H, int32_t N, int32_t d,
               int32_t G, const int32_t* off, int32_t Bk, int32_t C, int32_t iters, double scale,
               double tie_rel, double* mass, double* centroids, int32_t* counts, int32_t* ambiguous,
               int32_t nthreads) {
  const int32_t nK = (N + Bk - 1) / Bk;
  const int64_t BH = static_cast<int64_t>(B) * H;
  std::vector<double> kbar(static_cast<size_t>(BH) * nK * d);
  std::vector<int32_t> L(static_cast<size_t>(BH) * nK);
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic)
  for (int64_t bh = 0; bh < BH; ++bh)
    ref_key_means(k + bh * N * d, N, d, Bk, kbar.data() + bh * nK * d, L.data() + bh * nK);
#pragma omp parallel for schedule(dynamic)
  for (int64_t t = 0; t < BH * G; ++t) {
    const int64_t bh = t / G;
    const int32_t g = static_cast<int32_t>(t % G);
    const int32_t r0 = off[g], n = off[g + 1] - off[g];
    double* mu = centroids + t * C * d;
    int32_t* cnt = counts + t * C;
    const int32_t amb = ref_kmeans_group(q + (bh * N + r0) * d, n, d, C, iters, tie_rel, mu, cnt);
    if (ambiguous) ambiguous[t] = amb;
    ref_mass_group(mu, cnt, C, kbar.data() + bh * nK * d, L.data() + bh * nK, nK, d, scale,
                   mass + t * nK);
  }
}

// ---------------------------------------------------------------------------
// [AB] SIP / [IG] exact set + weighted sample, one plan row.
//
//  (1) Exact set E: the n_exact blocks of largest mass, ties to the lower
//      block index ("keep the highest-scoring blocks").  Mass is read as the
//      fp32 value the selector receives; non-finite or non-positive mass is
//      taken as 0 (a non-finite value also sets *bad).
//  (2) The rest R is sampled "in proportion to these estimates".  Weights are
//      quantised (reading): with m_max the largest mass in R,
//      w_b = floor(m_b / m_max * 2^31) + 1 (fp64 division, round to nearest),
//      or w_b = 1 for all b when m_max = 0.  The +1 keeps every pi > 0.
//  (3) "Highly scored blocks may always enter": inclusion probabilities
//      n' w_b / T are capped at 1 by the fixed-point iteration: repeat
//      { T = sum of w over R \ A; n' = n_s - |A|; move every b with
//      n' w_b >= T into A } until nothing moves.  A has pi = 1.
//  (4) "The sampler returns a fixed number of distinct blocks": systematic
//      PPS over the uncapped rest in ascending block order, n' points at
//      (i + u) T / n'; block j is drawn when a point falls in
//      [W_{j-1}, W_j) of the cumulative weights.  Done in exact integers:
//      f(x) = max(0, ceil((x n' 2^32 - U T) / (T 2^32))) counts the points
//      below x, and j is drawn iff f(W_j) - f(W_{j-1}) = 1.
//  (5) "A block sampled with probability one quarter counts four times": a
//      drawn block carries log_w = ln(1/pi) = ln T - ln(n' w_b), computed in
//      fp64 and stored as fp32; exact and capped blocks carry 0.
//  Plan row (reading): E ascending, then (A and the drawn blocks) ascending.
//  If n_sample >= |R| every block of R is included with log_w = 0.
//  pi (optional, [nK]): the inclusion probability of every block.
// Returns 0, or -1 on bad arguments.
// ---------------------------------------------------------------------------
int32_t ref_select_row(const float* mass, int32_t nK, int32_t n_exact, int32_t n_sample, uint32_t U,
                       int32_t* idx, float* log_w, double* pi, int32_t* bad) {
  if (n_exact < 0 || n_sample < 0 || n_exact + n_sample > nK) return -1;
  std::vector<uint32_t> key(nK);
  for (int32_t b = 0; b < nK; ++b) {
    const float m = mass[b];
    if (!std::isfinite(m)) {
      if (bad) *bad = 1;
      key[b] = 0;
    } else {
      key[b] = m > 0.0f ? float_bits(m) : 0u;  // positive floats order like their bit patterns
    }
  }
  std::vector<int32_t> order(nK);
  for (int32_t b = 0; b < nK; ++b) order[b] = b;
  std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
    return key[a] != key[b] ? key[a] > key[b] : a < b;
  });
  std::vector<char> in_exact(nK, 0);
  for (int32_t i = 0; i < n_exact; ++i) in_exact[order[i]] = 1;
  std::vector<double> p(nK, 0.0);
  std::vector<float> lw(nK, 0.0f);
  std::vector<char> chosen(nK, 0);
  std::vector<int32_t> rest;
  for (int32_t b = 0; b < nK; ++b) {
    if (in_exact[b]) {
      p[b] = 1.0;
    } else {
      rest.push_back(b);
    }
  }
  if (n_sample >= static_cast<int32_t>(rest.size())) {
    for (int32_t b : rest) {
      p[b] = 1.0;
      chosen[b] = 1;
    }
  } else if (n_sample > 0) {
    double m_max = 0.0;
    for (int32_t b : rest) m_max = std::max(m_max, static_cast<double>(bits_float(key[b])));
    std::vector<uint64_t> w(nK, 0);
    for (int32_t b : rest) {
      w[b] = m_max > 0.0
                 ? static_cast<uint64_t>(std::floor(static_cast<double>(bits_float(key[b])) / m_max * 2147483648.0)) + 1
                 : 1;
    }
    std::vector<char> capped(nK, 0);
    int32_t n_capped = 0;
    uint64_t T = 0;
    int64_t n_left = n_sample;
    for (;;) {
      T = 0;
      for (int32_t b : rest)
        if (!capped[b]) T += w[b];
      n_left = n_sample - n_capped;
      std::vector<int32_t> add;
      for (int32_t b : rest)
        if (!capped[b] && static_cast<u128>(n_left) * w[b] >= T) add.push_back(b);
      if (add.empty()) break;
      for (int32_t b : add) {
        capped[b] = 1;
        chosen[b] = 1;
        p[b] = 1.0;
      }
      n_capped += static_cast<int32_t>(add.size());
    }
    if (n_left > 0) {
      const u128 den = static_cast<u128>(T) << 32;
      const u128 uT = static_cast<u128>(U) * T;
      auto points_below = [&](uint64_t x) -> u128 {
        const u128 num = (static_cast<u128>(x) * static_cast<uint64_t>(n_left)) << 32;
        if (num <= uT) return 0;
        return (num - uT + den - 1) / den;
      };
      uint64_t W = 0;
      u128 f_prev = 0;
      for (int32_t b : rest) {
        if (capped[b]) continue;
        W += w[b];
        const u128 f = points_below(W);
        p[b] = static_cast<double>(static_cast<u128>(n_left) * w[b]) / static_cast<double>(T);
        if (f != f_prev) {
          chosen[b] = 1;
          lw[b] = static_cast<float>(std::log(static_cast<double>(T)) -
                                     std::log(static_cast<double>(static_cast<u128>(n_left) * w[b])));
        }
        f_prev = f;
      }
    }
  }
  int32_t s = 0;
  for (int32_t b = 0; b < nK; ++b)
    if (in_exact[b]) {
      idx[s] = b;
      log_w[s] = 0.0f;
      ++s;
    }
  for (int32_t b = 0; b < nK; ++b)
    if (chosen[b]) {
      idx[s] = b;
      log_w[s] = lw[b];
      ++s;
    }
  if (pi)
    for (int32_t b = 0; b < nK; ++b) pi[b] = p[b];
  return s == n_exact + n_sample ? 0 : -2;
}

// All plan rows of a [B, H, G, nK] fp32 mass tensor; idx / log_w: [B, H, G, S].
// Each row draws its own uniform from (seed, batch, head, group).
int32_t ref_select(const float* mass, int32_t B, int32_t H, int32_t G, int32_t nK, int32_t n_exact,
                   int32_t n_sample, uint64_t seed, int32_t* idx, float* log_w, int32_t* bad,
                   int32_t nthreads) {
  const int32_t S = n_exact + n_sample;
  const int64_t rows = static_cast<int64_t>(B) * H * G;
  int32_t status = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic) reduction(min : status)
  for (int64_t r = 0; r < rows; ++r) {
    const int32_t g = static_cast<int32_t>(r % G);
    const int32_t h = static_cast<int32_t>((r / G) % H);
    const int32_t b = static_cast<int32_t>(r / (static_cast<int64_t>(G) * H));
    const uint32_t U = ref_group_uniform(seed, b, h, g);
    int32_t row_bad = 0;
    const int32_t st = ref_select_row(mass + r * nK, nK, n_exact, n_sample, U, idx + r * S, log_w + r * S,
                                      nullptr, &row_bad);
    if (row_bad && bad) {
#pragma omp atomic write
      *bad = 1;
    }
    status = std::min(status, st);
  }
  return status;
}

// ---------------------------------------------------------------------------
// Exact-set size from a share of the mass (the top-p rule of "iCATS", Method
// summary: sparsity set by the share p of attention mass kept).  Reading: the
// exact set is the shortest head of the blocks in descending mass order (ties
// to the lower block) whose mass reaches the share p of the row's total; it is
// capped at the plan size S, and the rest of the budget, S - k_e, is sampled
// as above.  In exact integers, so that every implementation agrees:
//   q_b = floor(m_b / m_max * 2^31) in IEEE fp64 for m_b > 0, else 0
//         (m_max = the row's largest mass; all q are 0 when it is 0);
//   target = ceil(p * sum_b q_b) in fp64 (the sum is below 2^45: exact);
//   k_e = min(S, smallest k with q_(1) + ... + q_(k) >= target).
// A row of zeros has target 0 and k_e = 0.  Non-finite masses count as 0
// (and set *bad).  Returns k_e, or -1 on bad arguments.
// ---------------------------------------------------------------------------
int32_t ref_top_p_count(const float* mass, int32_t nK, double p, int32_t S, int32_t* bad) {
  if (nK < 1 || S < 0 || S > nK || !(p > 0.0) || p > 1.0) return -1;
  std::vector<uint32_t> key(nK);
  uint32_t kmax = 0;
  for (int32_t b = 0; b < nK; ++b) {
    const float m = mass[b];
    if (!std::isfinite(m)) {
      if (bad) *bad = 1;
      key[b] = 0;
    } else {
      key[b] = m > 0.0f ? float_bits(m) : 0u;
    }
    kmax = std::max(kmax, key[b]);
  }
  float mmax_f;
  std::memcpy(&mmax_f, &kmax, 4);
  const double mmax = static_cast<double>(mmax_f);
  std::vector<uint64_t> q(nK, 0);
  uint64_t total = 0;
  for (int32_t b = 0; b < nK; ++b) {
    if (key[b] != 0 && mmax > 0.0) {
      float f;
      std::memcpy(&f, &key[b], 4);
      q[b] = static_cast<uint64_t>(std::floor(static_cast<double>(f) / mmax * 2147483648.0));
    }
    total += q[b];
  }
  const uint64_t target = static_cast<uint64_t>(std::ceil(p * static_cast<double>(total)));
  // descending key, ties to the lower block
  std::vector<int32_t> order(nK);
  for (int32_t b = 0; b < nK; ++b) order[b] = b;
  std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) { return key[x] > key[y]; });
  int32_t k = 0;
  uint64_t cum = 0;
  while (cum < target && k < nK) cum += q[order[k++]];
  return std::min(k, S);
}

// All rows of a [B, H, G, nK] mass tensor under the top-p rule: the exact-set
// size of each row (k_e, [B, H, G]) and the plan with n_exact = k_e and
// n_sample = S - k_e (idx / log_w: [B, H, G, S]); uniforms as ref_select.
int32_t ref_select_top_p(const float* mass, int32_t B, int32_t H, int32_t G, int32_t nK, double p, int32_t S,
                         uint64_t seed, int32_t* idx, float* log_w, int32_t* k_e, int32_t* bad,
                         int32_t nthreads) {
  const int64_t rows = static_cast<int64_t>(B) * H * G;
  int32_t status = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic) reduction(min : status)
  for (int64_t r = 0; r < rows; ++r) {
    const int32_t g = static_cast<int32_t>(r % G);
    const int32_t h = static_cast<int32_t>((r / G) % H);
    const int32_t b = static_cast<int32_t>(r / (static_cast<int64_t>(G) * H));
    int32_t row_bad = 0;
    const int32_t ke = ref_top_p_count(mass + r * nK, nK, p, S, &row_bad);
    int32_t st = ke < 0 ? -1 : 0;
    if (st == 0) {
      k_e[r] = ke;
      st = ref_select_row(mass + r * nK, nK, ke, S - ke, ref_group_uniform(seed, b, h, g), idx + r * S,
                          log_w + r * S, nullptr, &row_bad);
    }
    if (row_bad && bad) {
#pragma omp atomic write
      *bad = 1;
    }
    status = std::min(status, st);
  }
  return status;
}

// ---------------------------------------------------------------------------
// [AB] the sparse pass: "the weights become shifts to the sampled attention
// scores before softmax ... only sampled blocks receive the exact attention
// computation".  For every query row of the listed groups:
//   z_k = scale * q . k + log_w(block of k)  over the valid rows of the plan's
//   blocks, O = sum_k e^{z_k - max} v_k / sum_k e^{z_k - max},
//   lse = max + ln sum_k e^{z_k - max}.
// With every block in the plan and log_w = 0 this is dense softmax attention.
// groups: n_list triples (batch, head, group).  out: [n_list rows...] packed
// in list order, each group's rows in row order, d values per row; lse
// likewise one value per row.
// ---------------------------------------------------------------------------
void ref_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int32_t B, int32_t H,
                   int32_t N, int32_t d, int32_t G, const int32_t* off, int32_t Bk, const int32_t* idx,
                   const float* log_w, int32_t S, double scale, const int32_t* groups, int32_t n_list,
                   double* out, double* lse, int32_t nthreads) {
  (void)B;
  std::vector<int64_t> base(n_list + 1, 0);
  for (int32_t i = 0; i < n_list; ++i) {
    const int32_t g = groups[3 * i + 2];
    base[i + 1] = base[i] + (off[g + 1] - off[g]);
  }
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic)
  for (int32_t i = 0; i < n_list; ++i) {
    const int32_t bb = groups[3 * i], h = groups[3 * i + 1], g = groups[3 * i + 2];
    const int64_t bh = static_cast<int64_t>(bb) * H + h;
    const int64_t prow = (bh * G + g) * S;
    std::vector<double> qrow(d), z, acc(d);
    std::vector<int64_t> keys;
    std::vector<double> bias;
    for (int32_t s = 0; s < S; ++s) {
      const int32_t blk = idx[prow + s];
      for (int32_t r = blk * Bk; r < std::min(N, (blk + 1) * Bk); ++r) {
        keys.push_back(r);
        bias.push_back(static_cast<double>(log_w[prow + s]));
      }
    }
    z.resize(keys.size());
    for (int32_t r = off[g]; r < off[g + 1]; ++r) {
      for (int32_t j = 0; j < d; ++j) qrow[j] = bf16_value(q[(bh * N + r) * d + j]);
      double mx = -INFINITY;
      for (size_t t = 0; t < keys.size(); ++t) {
        double dot = 0.0;
        const uint16_t* kr = k + (bh * N + keys[t]) * d;
        for (int32_t j = 0; j < d; ++j) dot += qrow[j] * bf16_value(kr[j]);
        z[t] = scale * dot + bias[t];
        mx = std::max(mx, z[t]);
      }
      double sum = 0.0;
      std::fill(acc.begin(), acc.end(), 0.0);
      for (size_t t = 0; t < keys.size(); ++t) {
        const double e = std::exp(z[t] - mx);
        sum += e;
        const uint16_t* vr = v + (bh * N + keys[t]) * d;
        for (int32_t j = 0; j < d; ++j) acc[j] += e * bf16_value(vr[j]);
      }
      const int64_t o = base[i] + (r - off[g]);
      for (int32_t j = 0; j < d; ++j) out[o * d + j] = acc[j] / sum;
      if (lse) lse[o] = mx + std::log(sum);
    }
  }
}

// Dense softmax attention softmax(scale Q K^T) V for the listed rows:
// rows: n_rows pairs (batch*H + head, row).  out: [n_rows, d]; lse: [n_rows].
void ref_dense_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int32_t N, int32_t d,
                         double scale, const int64_t* rows, int32_t n_rows, double* out, double* lse,
                         int32_t nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic)
  for (int32_t i = 0; i < n_rows; ++i) {
    const int64_t bh = rows[2 * i], r = rows[2 * i + 1];
    std::vector<double> qrow(d), z(N), acc(d, 0.0);
    for (int32_t j = 0; j < d; ++j) qrow[j] = bf16_value(q[(bh * N + r) * d + j]);
    double mx = -INFINITY;
    for (int32_t t = 0; t < N; ++t) {
      double dot = 0.0;
      const uint16_t* kr = k + (bh * N + t) * d;
      for (int32_t j = 0; j < d; ++j) dot += qrow[j] * bf16_value(kr[j]);
      z[t] = scale * dot;
      mx = std::max(mx, z[t]);
    }
    double sum = 0.0;
    for (int32_t t = 0; t < N; ++t) {
      const double e = std::exp(z[t] - mx);
      sum += e;
      const uint16_t* vr = v + (bh * N + t) * d;
      for (int32_t j = 0; j < d; ++j) acc[j] += e * bf16_value(vr[j]);
    }
    for (int32_t j = 0; j < d; ++j) out[static_cast<int64_t>(i) * d + j] = acc[j] / sum;
    if (lse) lse[i] = mx + std::log(sum);
  }
}

// ---------------------------------------------------------------------------
// [IG] / [AB] the permuted layout of permuted block-sparse attention: tokens
// of one (batch, head) are clustered over the whole sequence ("semantic-
// aware permutation", the SVG2 layout InstaGen is parameterised by) and
// reordered so that each cluster's rows are contiguous; a query cluster is
// then one query group and the reordered keys form the key blocks.
// (reading) Lloyd's k-means over the N rows of x with C clusters,
// centroids initialised at rows floor(c N / C), `iters` rounds of
//   assign  label_r = argmin_c ||x_r - mu_c||^2 (ties to the lower c),
//   sort    perm = the rows ordered by (label, row): a stable counting sort;
//           offsets[c] = number of rows with a label below c,
//   update  mu_c = mean of the rows of cluster c (an empty cluster keeps its
//           centroid),
// and the labels, permutation and offsets of the last round are the result.
// ---------------------------------------------------------------------------

// One assignment round.  x: [n, d] bf16 bits, mu: [C, d].  labels: [n].
// ambiguous (optional, [n]): 1 where the best and second-best squared
// distances differ by at most tie_rel * (||x||^2 + ||mu||^2), the margin
// below which a single-precision implementation may choose differently.
void ref_cluster_assign(const uint16_t* x, int32_t n, int32_t d, const double* mu, int32_t C, double tie_rel,
                        int32_t* labels, int32_t* ambiguous) {
  for (int32_t r = 0; r < n; ++r) {
    std::vector<double> xr(d);
    double xx = 0.0;
    for (int32_t j = 0; j < d; ++j) {
      xr[j] = bf16_value(x[static_cast<int64_t>(r) * d + j]);
      xx += xr[j] * xr[j];
    }
    double best = INFINITY, second = INFINITY, mm_best = 0.0, mm_second = 0.0;
    int32_t arg = 0;
    for (int32_t c = 0; c < C; ++c) {
      double dist = 0.0, mm = 0.0;
      for (int32_t j = 0; j < d; ++j) {
        const double m = mu[static_cast<int64_t>(c) * d + j];
        dist += (xr[j] - m) * (xr[j] - m);
        mm += m * m;
      }
      if (dist < best) {
        second = best;
        mm_second = mm_best;
        best = dist;
        mm_best = mm;
        arg = c;
      } else if (dist < second) {
        second = dist;
        mm_second = mm;
      }
    }
    labels[r] = arg;
    if (ambiguous) ambiguous[r] = (C > 1 && second - best <= tie_rel * (xx + std::max(mm_best, mm_second))) ? 1 : 0;
  }
}

// Stable counting sort of the labels: perm[i] = the i-th row in (label, row)
// order; offsets: [C + 1], offsets[c] .. offsets[c + 1] the rows of cluster c.
void ref_cluster_sort(const int32_t* labels, int32_t n, int32_t C, int32_t* perm, int32_t* offsets) {
  std::vector<int32_t> next(C + 1, 0);
  for (int32_t r = 0; r < n; ++r) next[labels[r] + 1] += 1;
  for (int32_t c = 0; c < C; ++c) next[c + 1] += next[c];
  for (int32_t c = 0; c <= C; ++c) offsets[c] = next[c];
  for (int32_t r = 0; r < n; ++r) perm[next[labels[r]]++] = r;
}

// Centroid update from the labels: mu_c = mean of its rows; counts: [C].
void ref_cluster_update(const uint16_t* x, int32_t n, int32_t d, const int32_t* labels, int32_t C, double* mu,
                        int32_t* counts) {
  std::vector<double> sum(static_cast<size_t>(C) * d, 0.0);
  for (int32_t c = 0; c < C; ++c) counts[c] = 0;
  for (int32_t r = 0; r < n; ++r) {
    counts[labels[r]] += 1;
    for (int32_t j = 0; j < d; ++j)
      sum[static_cast<int64_t>(labels[r]) * d + j] += bf16_value(x[static_cast<int64_t>(r) * d + j]);
  }
  for (int32_t c = 0; c < C; ++c) {
    if (counts[c] == 0) continue;
    for (int32_t j = 0; j < d; ++j) mu[static_cast<int64_t>(c) * d + j] = sum[static_cast<int64_t>(c) * d + j] / counts[c];
  }
}

// The whole clustering of every (batch, head): x [BH, N, d] bf16 bits.
// labels, perm: [BH, N]; offsets: [BH, C + 1]; mu: [BH, C, d];
// ambiguous: [BH] (1 if any round of that head met a near tie).
int32_t ref_cluster_tokens(const uint16_t* x, int32_t BH, int32_t N, int32_t d, int32_t C, int32_t iters,
                           double tie_rel, int32_t* labels, int32_t* perm, int32_t* offsets, double* mu,
                           int32_t* ambiguous, int32_t nthreads) {
  if (BH < 1 || N < 1 || d < 1 || C < 1 || C > N || iters < 1) return -1;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic)
  for (int32_t bh = 0; bh < BH; ++bh) {
    const uint16_t* xb = x + static_cast<int64_t>(bh) * N * d;
    double* mub = mu + static_cast<int64_t>(bh) * C * d;
    int32_t* lab = labels + static_cast<int64_t>(bh) * N;
    for (int32_t c = 0; c < C; ++c) {
      const int64_t r = (static_cast<int64_t>(c) * N) / C;
      for (int32_t j = 0; j < d; ++j) mub[static_cast<int64_t>(c) * d + j] = bf16_value(xb[r * d + j]);
    }
    std::vector<int32_t> amb(N), counts(C);
    int32_t any = 0;
    for (int32_t it = 0; it < iters; ++it) {
      ref_cluster_assign(xb, N, d, mub, C, tie_rel, lab, amb.data());
      for (int32_t r = 0; r < N; ++r) any |= amb[r];
      ref_cluster_update(xb, N, d, lab, C, mub, counts.data());
    }
    ref_cluster_sort(lab, N, C, perm + static_cast<int64_t>(bh) * N, offsets + static_cast<int64_t>(bh) * (C + 1));
    ambiguous[bh] = any;
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Tail merging of the permuted layout.  [IC] "Approach": the tail blocks of
// query clusters are merged with Hamming-nearest compatible clusters, to cut
// the padding of their last tiles.  Readings:
//  * the tail of cluster g is its last t_g = n_g mod 128 rows (all of it when
//    n_g < 128; no tail when t_g = 0); in a merged 128-row tile it takes a slot
//    of ceil(t_g / 32) * 32 rows (whole quarters of the tile, so that the
//    rows a tile's softmax handles together share one plan), members packed
//    from row 0 in the order they joined;
//  * tails are taken in order of decreasing t_g, ties to the lower g;
//  * a tail is compatible with an open tile when its slot fits in the rows
//    left, the tile has fewer than 4 members, and the union U of the members'
//    plan blocks, with the tail's plan P added, needs fewer KV tiles of
//    128 / Bk blocks than U and P apart: ceil(|U u P| / b) < ceil(|U| / b) +
//    ceil(|P| / b);
//  * it joins the compatible tile whose union is Hamming-nearest to P
//    (|U xor P| smallest, ties to the tile opened first), else opens a tile;
//  * every row keeps its own cluster's plan and log-weights: the merged tile
//    runs the blocks of U in ascending order, and a block outside a row's plan
//    is masked for that row, so each row's attention is unchanged.
// One (batch, head): off [G+1], idx [G][S] (that head's plan rows).  Outputs,
// one entry per tile in the order the tiles were opened: members[t][4] (the
// clusters, -1 past the last), slots[t][4] (first row of each member's slot),
// ulen[t] and units[t][4 S] (U ascending).  Returns the number of tiles.
int32_t ref_tail_merge(const int32_t* off, int32_t G, const int32_t* idx, int32_t S, int32_t Bk,
                       int32_t* members, int32_t* slots, int32_t* ulen, int32_t* units) {
  const int32_t b = 128 / Bk;
  auto tiles_of = [&](int64_t n) { return (n + b - 1) / b; };
  struct Tail {
    int32_t g, t;
  };
  std::vector<Tail> tails;
  for (int32_t g = 0; g < G; ++g) {
    const int32_t t = (off[g + 1] - off[g]) % 128;
    if (t > 0) tails.push_back({g, t});
  }
  std::stable_sort(tails.begin(), tails.end(), [](const Tail& x, const Tail& y) { return x.t > y.t; });
  struct Tile {
    int32_t rows, n;
    int32_t g[4], slot[4];
    std::vector<int32_t> u;  // ascending
  };
  std::vector<Tile> tiles;
  for (const Tail& tl : tails) {
    std::vector<int32_t> p(idx + static_cast<int64_t>(tl.g) * S, idx + static_cast<int64_t>(tl.g + 1) * S);
    std::sort(p.begin(), p.end());
    const int32_t rows = (tl.t + 31) / 32 * 32;
    int32_t best = -1;
    int64_t best_h = 0;
    std::vector<int32_t> best_u;
    for (size_t i = 0; i < tiles.size(); ++i) {
      const Tile& tt = tiles[i];
      if (tt.rows + rows > 128 || tt.n >= 4) continue;
      std::vector<int32_t> un;
      std::set_union(tt.u.begin(), tt.u.end(), p.begin(), p.end(), std::back_inserter(un));
      if (tiles_of(static_cast<int64_t>(un.size())) >=
          tiles_of(static_cast<int64_t>(tt.u.size())) + tiles_of(static_cast<int64_t>(p.size())))
        continue;
      const int64_t inter = static_cast<int64_t>(tt.u.size() + p.size() - un.size());
      const int64_t ham = static_cast<int64_t>(tt.u.size() + p.size()) - 2 * inter;
      if (best < 0 || ham < best_h) {
        best = static_cast<int32_t>(i);
        best_h = ham;
        best_u = un;
      }
    }
    if (best < 0) {
      Tile tt;
      tt.rows = rows;
      tt.n = 1;
      tt.g[0] = tl.g;
      tt.slot[0] = 0;
      tt.u = p;
      tiles.push_back(tt);
    } else {
      Tile& tt = tiles[best];
      tt.g[tt.n] = tl.g;
      tt.slot[tt.n] = tt.rows;
      ++tt.n;
      tt.rows += rows;
      tt.u = best_u;
    }
  }
  for (size_t i = 0; i < tiles.size(); ++i) {
    for (int32_t m = 0; m < 4; ++m) {
      members[4 * i + m] = m < tiles[i].n ? tiles[i].g[m] : -1;
      slots[4 * i + m] = m < tiles[i].n ? tiles[i].slot[m] : -1;
    }
    ulen[i] = static_cast<int32_t>(tiles[i].u.size());
    std::copy(tiles[i].u.begin(), tiles[i].u.end(), units + static_cast<int64_t>(i) * 4 * S);
  }
  return static_cast<int32_t>(tiles.size());
}

int32_t ref_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
