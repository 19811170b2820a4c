// Dynamic block size (host code): the acceptance counts of each sequence and the choice
// of K that commits the most tokens per unit time. The pages leave K to future work and
// suggest choosing it by how certain the generation is (news article, "Future
// Directions: Larger K and Higher Acceptance", item 1); certainty is read here as the
// per-position acceptance rate alpha of a geometric acceptance process:
//   P(a >= j) = alpha^j for j <= K,  so  E[a + 1 | K] = sum_{j=0..K} alpha^j.
#pragma once
#include <cmath>

#include "orthrus.h"

namespace orthrus {

// sum_{j=0..K} alpha^j in double, by the closed form away from alpha = 1
inline double expected_committed(double alpha, int K) {
  if (alpha >= 1.0) return (double)(K + 1);
  if (alpha <= 0.0) return 1.0;
  return (1.0 - std::pow(alpha, (double)(K + 1))) / (1.0 - alpha);
}

inline double accept_rate(const orthrus_accept_stats& s) {
  return ((double)s.accepted + 1.0) / ((double)s.accepted + (double)s.rejected + 2.0);
}

}  // namespace orthrus

extern "C" {

orthrus_status orthrus_accept_stats_update(orthrus_accept_stats* stats, const int32_t* accept_len, int32_t batch,
                                           int32_t K, float decay) {
  if (!stats || !accept_len || batch < 1 || K < 0 || K > 64 || !(decay > 0.f && decay <= 1.f)) return ORTHRUS_ERR_ARG;
  for (int b = 0; b < batch; ++b)
    if (accept_len[b] > K) return ORTHRUS_ERR_ARG;
  for (int b = 0; b < batch; ++b) {
    const int a = accept_len[b];
    if (a < 0) continue;  // a failed step commits nothing and says nothing about alpha
    stats[b].accepted = decay * stats[b].accepted + (float)a;
    stats[b].rejected = decay * stats[b].rejected + (a < K ? 1.f : 0.f);
  }
  return ORTHRUS_OK;
}

float orthrus_accept_rate(const orthrus_accept_stats* stats) {
  if (!stats || stats->accepted < 0.f || stats->rejected < 0.f) return -1.f;
  return (float)orthrus::accept_rate(*stats);
}

int32_t orthrus_choose_block_size(const orthrus_accept_stats* stats, int32_t batch, const int32_t* ks,
                                  const float* step_ms, int32_t n_options) {
  if (!stats || !ks || !step_ms || batch < 1 || n_options < 1) return -1;
  for (int i = 0; i < n_options; ++i)
    if (ks[i] < 1 || ks[i] > 64 || !(step_ms[i] > 0.f)) return -1;
  for (int b = 0; b < batch; ++b)
    if (stats[b].accepted < 0.f || stats[b].rejected < 0.f) return -1;
  int best_k = -1;
  double best = -1.0;
  for (int i = 0; i < n_options; ++i) {
    double tokens = 0.0;
    for (int b = 0; b < batch; ++b) tokens += orthrus::expected_committed(orthrus::accept_rate(stats[b]), ks[i]);
    const double rate = tokens / (double)step_ms[i];
    if (rate > best || (rate == best && ks[i] < best_k)) {
      best = rate;
      best_k = ks[i];
    }
  }
  return best_k;
}

}  // extern "C"
