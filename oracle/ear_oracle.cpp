// SVG-EAR CPU oracle: plain, slow, fp64 restatement of the attention hot path.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// benchmark's CPU-baseline / reference arm may load this library.  It shares
// no code with the CUDA path: no headers, no helpers, no tables.
//
// Citations ("SVG-EAR §x") refer to the paper "SVG-EAR: Parameter-Free Linear
// Compensation for Sparse Video Generation via Error-aware Routing"
// (arXiv 2603.08982), by section.  Where the pages leave a step open the
// reading taken is stated beside the code.
//
// Every function works on ONE (batch, head) slice, in original token order,
// with inputs already upcast to double.  Matrices are row-major [rows][d].
//
// Parity status: every function here is pinned by CPU tests (closed forms,
// scipy's Lloyd k-means, a token-level numpy brute force and a hand-worked
// example); none is "parity unpinned".

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// ---------------------------------------------------------------------------
// Step 1: k-means (SVG-EAR §4.1 Problem Formulation: Q and K are clustered
// with "flash k-means" into C_q and C_k clusters; q̄_i / k̄_j is the mean
// token of the cluster holding i / j).
//
// Reading: "flash k-means" is named, not defined, so this is plain Euclidean
// Lloyd iteration from a given initial centroid set.  Each of `iters`
// iterations assigns every row to argmin_c sum_k (x_k - c_k)^2 (written out
// as a sum of squared differences; ties go to the lowest c), then moves every
// centroid to the mean of its members; an empty cluster keeps its previous
// centroid.  Labels come from the last assignment and the returned centroids
// are the means of those final members ("the mean token in the cluster").
// ---------------------------------------------------------------------------
void oracle_kmeans(const double* X, int64_t N, int32_t d, int32_t C, int32_t iters,
                   const double* init, double* centroids, int32_t* labels,
                   int64_t* counts) {
  std::memcpy(centroids, init, sizeof(double) * (size_t)C * d);
  std::vector<double> sums((size_t)C * d);
  for (int32_t t = 0; t < iters; ++t) {
    // assignment
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
      const double* x = X + i * d;
      int32_t best = 0;
      double best_dist = std::numeric_limits<double>::infinity();
      for (int32_t c = 0; c < C; ++c) {
        const double* cc = centroids + (size_t)c * d;
        double dist = 0.0;
        for (int32_t k = 0; k < d; ++k) {
          double diff = x[k] - cc[k];
          dist += diff * diff;
        }
        if (dist < best_dist) {  // strict: the first (lowest) index wins ties
          best_dist = dist;
          best = c;
        }
      }
      labels[i] = best;
    }
    // update: member means, rows summed in token order
    std::fill(sums.begin(), sums.end(), 0.0);
    std::fill(counts, counts + C, (int64_t)0);
    for (int64_t i = 0; i < N; ++i) {
      int32_t c = labels[i];
      counts[c] += 1;
      for (int32_t k = 0; k < d; ++k) sums[(size_t)c * d + k] += X[i * d + k];
    }
    for (int32_t c = 0; c < C; ++c) {
      if (counts[c] == 0) continue;  // empty cluster keeps its centroid
      for (int32_t k = 0; k < d; ++k)
        centroids[(size_t)c * d + k] = sums[(size_t)c * d + k] / (double)counts[c];
    }
  }
}

// ---------------------------------------------------------------------------
// Step 2: permutation (SVG-EAR §3.1: semantically similar tokens are
// clustered and permuted so each cluster is laid out contiguously, turning
// the attention map into (query cluster x key cluster) blocks).
//
// Reading: a stable sort of token indices by cluster label.  perm[r] is the
// original index of the token at permuted position r; offsets[c] is the first
// permuted position of cluster c (offsets[C] = N).
// ---------------------------------------------------------------------------
void oracle_permute(const int32_t* labels, int64_t N, int32_t C, int32_t* perm,
                    int64_t* offsets) {
  std::vector<int64_t> order(N);
  std::iota(order.begin(), order.end(), (int64_t)0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int64_t a, int64_t b) { return labels[a] < labels[b]; });
  for (int64_t r = 0; r < N; ++r) perm[r] = (int32_t)order[r];
  std::fill(offsets, offsets + C + 1, (int64_t)0);
  for (int64_t i = 0; i < N; ++i) offsets[labels[i] + 1] += 1;
  for (int32_t c = 0; c < C; ++c) offsets[c + 1] += offsets[c];
}

// Mean of the rows of X in each cluster (SVG-EAR §4.3 Linear Compensation:
// V follows the key clustering and v̄_j is the average of V over the key
// cluster holding j).  Empty clusters get a zero row (never used).
void oracle_segment_mean(const double* X, const int32_t* labels, int64_t N, int32_t d,
                         int32_t C, double* mean) {
  std::vector<int64_t> cnt(C, 0);
  std::fill(mean, mean + (size_t)C * d, 0.0);
  for (int64_t i = 0; i < N; ++i) {
    int32_t c = labels[i];
    cnt[c] += 1;
    for (int32_t k = 0; k < d; ++k) mean[(size_t)c * d + k] += X[i * d + k];
  }
  for (int32_t c = 0; c < C; ++c)
    if (cnt[c] > 0)
      for (int32_t k = 0; k < d; ++k) mean[(size_t)c * d + k] /= (double)cnt[c];
}

// ---------------------------------------------------------------------------
// Step 3: error probe (SVG-EAR §4.2 "Error estimation", §1 Introduction:
// query centroids stand in for the individual queries, so the estimate costs
// O(C_q N_k d) instead of O(N_q N_k d)).
//
// For query cluster a and key cluster b the per-entry estimate of key j in b
// is (s q̄_a·k_j - s q̄_a·k̄_b)^2: the gap between the exact logit and the
// compensated logit that replaces k_j by its centroid (SVG-EAR §3.1 / §4.1,
// logit q k̄ / sqrt(d)).  E[a][b] sums it over the keys of b.  Blocks with an
// empty query or key cluster get 0.  The per-entry equation itself is lost in
// the extracted pages; this logit-space form is the reading used here.
// ---------------------------------------------------------------------------
void oracle_probe(const double* q_cent, const int64_t* q_counts, const double* K,
                  const int32_t* k_labels, const double* k_cent, const int64_t* k_counts,
                  int64_t N_k, int32_t d, int32_t C_q, int32_t C_k, double scale,
                  double* E) {
#pragma omp parallel for schedule(dynamic)
  for (int32_t a = 0; a < C_q; ++a) {
    double* row = E + (size_t)a * C_k;
    for (int32_t b = 0; b < C_k; ++b) row[b] = 0.0;
    if (q_counts[a] == 0) continue;
    const double* qa = q_cent + (size_t)a * d;
    std::vector<double> centroid_logit(C_k);
    for (int32_t b = 0; b < C_k; ++b) {
      double dot = 0.0;
      for (int32_t k = 0; k < d; ++k) dot += qa[k] * k_cent[(size_t)b * d + k];
      centroid_logit[b] = scale * dot;
    }
    for (int64_t j = 0; j < N_k; ++j) {
      int32_t b = k_labels[j];
      double dot = 0.0;
      for (int32_t k = 0; k < d; ++k) dot += qa[k] * K[j * d + k];
      double gap = scale * dot - centroid_logit[b];
      row[b] += gap * gap;
    }
    for (int32_t b = 0; b < C_k; ++b)
      if (k_counts[b] == 0) row[b] = 0.0;
  }
}

// ---------------------------------------------------------------------------
// Step 3, variants: error probes on the unnormalized attention weights
// (SVG-EAR §4.2 "Relaxed optimization problem": the relaxed objective
// compares unnormalized attention weights; §4.3: a value-aware estimate that
// also uses v_j and v̄_j, at the same O(C_q N_k d) cost; §4.4: the streaming
// kernel subtracts the running maximum of the logits before exponentiating).
//
// Reading (the per-entry equations are lost in the extracted pages): for query
// cluster a, z_j = s q̄_a·k_j, z̄_b = s q̄_a·k̄_b, m_a = max over every key j of
// the slice of z_j (the running maximum at the end of the stream), w_j =
// e^{z_j - m_a}, w̄_b = e^{z̄_b - m_a}; for key cluster b
//   mode 1 (weights):      E[a][b] = sum_{j in b} (w_j - w̄_b)^2
//   mode 2 (value-aware):  E[a][b] = sum_{j in b} || w_j v_j - w̄_b v̄_b ||^2
// Blocks with an empty query or key cluster get 0.
// ---------------------------------------------------------------------------
void oracle_probe_weights(const double* q_cent, const int64_t* q_counts, const double* K,
                          const int32_t* k_labels, const double* k_cent,
                          const int64_t* k_counts, const double* V, const double* v_cent,
                          int64_t N_k, int32_t d, int32_t C_q, int32_t C_k, double scale,
                          int32_t mode, double* E) {
#pragma omp parallel for schedule(dynamic)
  for (int32_t a = 0; a < C_q; ++a) {
    double* row = E + (size_t)a * C_k;
    for (int32_t b = 0; b < C_k; ++b) row[b] = 0.0;
    if (q_counts[a] == 0) continue;
    const double* qa = q_cent + (size_t)a * d;
    std::vector<double> z(N_k), zbar(C_k);
    double m = -std::numeric_limits<double>::infinity();
    for (int64_t j = 0; j < N_k; ++j) {
      double dot = 0.0;
      for (int32_t k = 0; k < d; ++k) dot += qa[k] * K[j * d + k];
      z[j] = scale * dot;
      m = std::max(m, z[j]);
    }
    for (int32_t b = 0; b < C_k; ++b) {
      double dot = 0.0;
      for (int32_t k = 0; k < d; ++k) dot += qa[k] * k_cent[(size_t)b * d + k];
      zbar[b] = scale * dot;
    }
    for (int64_t j = 0; j < N_k; ++j) {
      const int32_t b = k_labels[j];
      const double w = std::exp(z[j] - m), wbar = std::exp(zbar[b] - m);
      if (mode == 1) {
        const double g = w - wbar;
        row[b] += g * g;
      } else {
        double sq = 0.0;
        for (int32_t k = 0; k < d; ++k) {
          const double g = w * V[j * d + k] - wbar * v_cent[(size_t)b * d + k];
          sq += g * g;
        }
        row[b] += sq;
      }
    }
    for (int32_t b = 0; b < C_k; ++b)
      if (k_counts[b] == 0) row[b] = 0.0;
  }
}

// ---------------------------------------------------------------------------
// Step 4: greedy error-to-cost routing (SVG-EAR §4.2 "Error estimation":
// blocks are taken for exact attention in decreasing order of
// sum_{(i,j) in block} eps_ij^2 / (|q_c| |k_c|) until the budget is spent;
// §4.1: the budget is nnz(M) <= rho N_q N_k).
//
// mode 0 (the pages' ratio): the block sum of per-entry estimates is
//   |a| * E[a][b] because every query of a uses the same centroid, so the
//   ratio is E[a][b] / |b|.
// mode 1: E[a][b] / (|a| |b|), the literal "E over block size" form.
// Budget B = floor(rho * (N_q * N_k)) (product exact in int64, then double).
// Order: ratio descending, ties to the lower linear index a*C_k + b.  Blocks
// with |a||b| = 0 are never exact.  Walk the order adding |a||b| while the
// total stays <= B; stop at the first block that does not fit.
// exact_pairs receives the number of exact (query, key) pairs.
// ---------------------------------------------------------------------------
void oracle_route(const double* E, const int64_t* q_counts, const int64_t* k_counts,
                  int32_t C_q, int32_t C_k, int64_t N_q, int64_t N_k, double density,
                  int32_t mode, uint8_t* exact, int64_t* exact_pairs) {
  const int64_t total = N_q * N_k;
  const int64_t budget = (int64_t)std::floor(density * (double)total);
  struct Item { double ratio; int64_t index; int64_t cost; };
  std::vector<Item> items;
  items.reserve((size_t)C_q * C_k);
  for (int32_t a = 0; a < C_q; ++a)
    for (int32_t b = 0; b < C_k; ++b) {
      int64_t cost = q_counts[a] * k_counts[b];
      exact[(size_t)a * C_k + b] = 0;
      if (cost == 0) continue;
      double e = E[(size_t)a * C_k + b];
      double ratio = (mode == 0) ? e / (double)k_counts[b] : e / (double)cost;
      items.push_back({ratio, (int64_t)a * C_k + b, cost});
    }
  std::sort(items.begin(), items.end(), [](const Item& x, const Item& y) {
    if (x.ratio != y.ratio) return x.ratio > y.ratio;
    return x.index < y.index;
  });
  int64_t used = 0;
  for (const Item& it : items) {
    if (used + it.cost > budget) break;
    used += it.cost;
    exact[it.index] = 1;
  }
  *exact_pairs = used;
}

// ---------------------------------------------------------------------------
// Step 4, per query cluster (SVG-EAR §5 "Implementation": SVG2 gives every
// query cluster an adaptive budget, so the routing runs for each query
// cluster on its own).
//
// oracle_route_rows: for query cluster a with budget row_budget[a] (pairs),
// its blocks with |a||b| > 0 are walked in decreasing E[a][b] / |b| (within a
// query cluster this is also the order of E / (|a||b|)), ties to the lower b,
// adding |a||b| while the total stays <= row_budget[a] and stopping at the
// first block that does not fit.  pairs[a] receives the pairs taken.
//
// oracle_topp_budget (reading of SVG2's top-p budget, the score-based
// selection of SVG-EAR Fig. 2(c)): the key clusters' centroid attention mass
// for query cluster a is w_b = |b| e^{s q̄_a·k̄_b - max} over non-empty b;
// sorted by decreasing w (ties to the lower b), the smallest prefix whose
// cumulative mass reaches p times the total is the top-p set, and the budget
// is |a| times the key count of that set (0 for an empty query cluster).
// ---------------------------------------------------------------------------
void oracle_route_rows(const double* E, const int64_t* q_counts, const int64_t* k_counts,
                       int32_t C_q, int32_t C_k, const int64_t* row_budget, uint8_t* exact,
                       int64_t* pairs) {
  struct Item { double ratio; int32_t b; int64_t cost; };
  for (int32_t a = 0; a < C_q; ++a) {
    std::vector<Item> items;
    for (int32_t b = 0; b < C_k; ++b) {
      exact[(size_t)a * C_k + b] = 0;
      const int64_t cost = q_counts[a] * k_counts[b];
      if (cost == 0) continue;
      items.push_back({E[(size_t)a * C_k + b] / (double)k_counts[b], b, cost});
    }
    std::sort(items.begin(), items.end(), [](const Item& x, const Item& y) {
      if (x.ratio != y.ratio) return x.ratio > y.ratio;
      return x.b < y.b;
    });
    int64_t used = 0;
    for (const Item& it : items) {
      if (used + it.cost > row_budget[a]) break;
      used += it.cost;
      exact[(size_t)a * C_k + it.b] = 1;
    }
    pairs[a] = used;
  }
}

void oracle_topp_budget(const double* q_cent, const int64_t* q_counts, const double* k_cent,
                        const int64_t* k_counts, int32_t C_q, int32_t C_k, int32_t d,
                        double scale, double p, int64_t* budget) {
  for (int32_t a = 0; a < C_q; ++a) {
    budget[a] = 0;
    if (q_counts[a] == 0) continue;
    std::vector<double> z(C_k, -std::numeric_limits<double>::infinity());
    double zmax = -std::numeric_limits<double>::infinity();
    for (int32_t b = 0; b < C_k; ++b) {
      if (k_counts[b] == 0) continue;
      double dot = 0.0;
      for (int32_t k = 0; k < d; ++k) dot += q_cent[(size_t)a * d + k] * k_cent[(size_t)b * d + k];
      z[b] = scale * dot;
      zmax = std::max(zmax, z[b]);
    }
    std::vector<std::pair<double, int32_t>> w;
    double total = 0.0;
    for (int32_t b = 0; b < C_k; ++b) {
      if (k_counts[b] == 0) continue;
      const double m = (double)k_counts[b] * std::exp(z[b] - zmax);
      w.push_back({m, b});
      total += m;
    }
    std::sort(w.begin(), w.end(), [](const std::pair<double, int32_t>& x,
                                     const std::pair<double, int32_t>& y) {
      if (x.first != y.first) return x.first > y.first;
      return x.second < y.second;
    });
    double cum = 0.0;
    int64_t keys = 0;
    for (const auto& it : w) {
      if (cum >= p * total) break;  // the prefix already reaches p
      cum += it.first;
      keys += k_counts[it.second];
    }
    budget[a] = q_counts[a] * keys;
  }
}

// ---------------------------------------------------------------------------
// Step 5: block-sparse attention with linear compensation (SVG-EAR §4.1
// routing mask, §4.3 Linear Compensation, §3.1).
//
// The mask M is shared by all queries of a query cluster and by all keys of a
// key cluster.  For query i in cluster a, key j in cluster b:
//   exact block (M=1): logit s q_i·k_j with value v_j;
//   skipped block (M=0): logit s q_i·k̄_b with value v̄_b, the same for all
//   |b| keys of the cluster, so the cluster contributes |b| e^{logit} v̄_b.
// One softmax normalizer spans both kinds of terms.  With compensate = 0 the
// skipped blocks are dropped instead (the score-routed baseline of §3.1).
// O is written in original token order; lse = m + ln(L) (natural log).
// ---------------------------------------------------------------------------
void oracle_attention(const double* Q, const double* K, const double* V,
                      const int32_t* q_labels, const int32_t* k_labels,
                      const double* k_cent, const double* v_cent, const int64_t* k_counts,
                      const uint8_t* exact, int64_t N_q, int64_t N_k, int32_t d,
                      int32_t C_q, int32_t C_k, double scale, int32_t compensate,
                      double* O, double* lse) {
  (void)C_q;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t i = 0; i < N_q; ++i) {
    const double* q = Q + i * d;
    const uint8_t* mrow = exact + (size_t)q_labels[i] * C_k;
    std::vector<double> logit(N_k), clogit(C_k);
    double m = -std::numeric_limits<double>::infinity();
    for (int64_t j = 0; j < N_k; ++j) {
      if (!mrow[k_labels[j]]) continue;
      double dot = 0.0;
      for (int32_t k = 0; k < d; ++k) dot += q[k] * K[j * d + k];
      logit[j] = scale * dot;
      m = std::max(m, logit[j]);
    }
    if (compensate) {
      for (int32_t b = 0; b < C_k; ++b) {
        if (mrow[b] || k_counts[b] == 0) continue;
        double dot = 0.0;
        for (int32_t k = 0; k < d; ++k) dot += q[k] * k_cent[(size_t)b * d + k];
        clogit[b] = scale * dot;
        m = std::max(m, clogit[b]);
      }
    }
    double* o = O + i * d;
    for (int32_t k = 0; k < d; ++k) o[k] = 0.0;
    double L = 0.0;
    for (int64_t j = 0; j < N_k; ++j) {
      if (!mrow[k_labels[j]]) continue;
      double w = std::exp(logit[j] - m);
      L += w;
      for (int32_t k = 0; k < d; ++k) o[k] += w * V[j * d + k];
    }
    if (compensate) {
      for (int32_t b = 0; b < C_k; ++b) {
        if (mrow[b] || k_counts[b] == 0) continue;
        double w = (double)k_counts[b] * std::exp(clogit[b] - m);
        L += w;
        for (int32_t k = 0; k < d; ++k) o[k] += w * v_cent[(size_t)b * d + k];
      }
    }
    if (L > 0.0) {
      for (int32_t k = 0; k < d; ++k) o[k] /= L;
      lse[i] = m + std::log(L);
    } else {  // no term at all (only possible when nothing is exact and compensation is off)
      lse[i] = -std::numeric_limits<double>::infinity();
    }
  }
}

// ---------------------------------------------------------------------------
// Diagnostics (SVG-EAR §4.2 after "Error estimation": the bound's residual
// 8 δ_q^2 K_max^2 / (N_k d) grows with the clustering error δ_q^2; §5.3
// "Effect of clustering": δ_q^2 against the number of query centroids; §5.1:
// the average relative change of the softmax normalizer).
//
// Readings: δ^2 = (1/N) sum_i ||x_i - c_{l_i}||^2, the mean squared distance
// of the rows to their centroids (the k-means objective over N); K_max =
// max_j ||k_j||.  The normalizer change of query i is |Z_sparse / Z_dense - 1|
// with Z = e^{lse}, averaged over the queries.
// ---------------------------------------------------------------------------
void oracle_cluster_stats(const double* X, const int32_t* labels, const double* centroids,
                          int64_t N, int32_t d, double* mean_sq_dist, double* max_norm) {
  double sum = 0.0, mx = 0.0;
  for (int64_t i = 0; i < N; ++i) {
    const double* x = X + i * d;
    const double* c = centroids + (size_t)labels[i] * d;
    double dist = 0.0, nrm = 0.0;
    for (int32_t k = 0; k < d; ++k) {
      const double diff = x[k] - c[k];
      dist += diff * diff;
      nrm += x[k] * x[k];
    }
    sum += dist;
    mx = std::max(mx, std::sqrt(nrm));
  }
  *mean_sq_dist = N > 0 ? sum / (double)N : 0.0;
  *max_norm = mx;
}

double oracle_normalizer_change(const double* lse_sparse, const double* lse_dense, int64_t N) {
  double sum = 0.0;
  for (int64_t i = 0; i < N; ++i) {
    if (lse_sparse[i] == lse_dense[i]) continue;  // also both -inf: no change
    sum += std::fabs(std::exp(lse_sparse[i] - lse_dense[i]) - 1.0);
  }
  return N > 0 ? sum / (double)N : 0.0;
}

int32_t oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
