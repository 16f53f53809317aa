// Reference oracle for block-sparse GQA attention with a mean-pooled block cache.
//
// TEST INFRASTRUCTURE ONLY. This file is a plain, slow, fp64 CPU statement of
// what the method computes. Only the test suite, the smoke check and the
// benchmark's CPU-baseline leg may load it. It shares no code, header, table
// or helper with the CUDA library, and it never sees paged memory: every
// tensor here is logical and unpaged, so paging mistakes in the library show
// up as mismatches.
//
// The method (MoBA-style block sparsity with GQA-shared selection and a block
// cache) is described on:
//   * "Art of Focus: Ling 2.0 and the Revolution in Sparse Attention for
//     Ultra-Long Contexts" (undercodenews), section "Summarizing the
//     Breakthrough": keys and values are split into blocks, each query keeps
//     only its top-k blocks, the heads of a GQA group share one selection, and
//     blocks are aggregated into representations stored in a block cache.
//   * "MiniMax Sparse Attention" (staik.se), method and results paragraphs: an
//     index branch scores KV blocks and picks a top-k subset per GQA group with
//     an exp-free selection; exact attention then runs over the selected blocks.
//   * "Sparse Attention + Linear Backbones" (Baidu 9584117), section 5.5: the
//     attention over the selected set is softmax(q k_sel^T / sqrt(d)) v_sel.
// Where the pages are silent, the readings used here are:
//   * the block representation is the arithmetic mean of the block's keys,
//     over the tokens present;
//   * the score of block j for a query row and KV group g is
//     sum over the group's heads h of q_h . c_j (no scale, no softmax);
//   * candidates are complete past blocks j < b(t) = floor(t / B); the query's
//     own block b(t) is always selected, future blocks never; k counts the own
//     block, so the row keeps min(k, b(t)+1) blocks;
//   * ties in score go to the lower block index;
//   * inside the own block attention is token-causal (key position <= t);
//   * query head h belongs to KV group floor(h / G), G = Hq / Hkv.
//
// Element storage: dtype 0 = fp32, dtype 1 = bf16 bit patterns (uint16).
// Every element is widened to double on use.

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

double elem(const void* p, int dtype, int64_t i) {
  if (dtype == 0) return (double)((const float*)p)[i];
  uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return (double)f;
}

}  // namespace

extern "C" {

// Block representations: C[j][g][i] = mean over tokens u in block j that are
// present (u < L) of K[u][g][i]. Returns the number of blocks ceil(L / B).
int64_t orc_centroids(const void* K, int dtype, int64_t L, int hkv, int d, int B, double* C) {
  const int64_t nblk = (L + B - 1) / B;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < nblk; ++j) {
    const int64_t u0 = j * B;
    const int64_t u1 = std::min<int64_t>(u0 + B, L);
    const double n = (double)(u1 - u0);
    for (int g = 0; g < hkv; ++g) {
      for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int64_t u = u0; u < u1; ++u) s += elem(K, dtype, (u * hkv + g) * (int64_t)d + i);
        C[(j * hkv + g) * (int64_t)d + i] = s / n;
      }
    }
  }
  return nblk;
}

// Block scores: S[r][g][j] = sum_{h in group g} sum_i Q[r][h][i] * C[j][g][i]
// for candidate blocks j < floor(pos[r] / B); every other entry is NaN.
void orc_scores(const void* Q, int dtype, int64_t R, const int64_t* pos, int hq, int hkv, int d,
                int B, const double* C, int64_t nblk, double* S) {
  const int G = hq / hkv;
  const double nan = std::numeric_limits<double>::quiet_NaN();
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < R; ++r) {
    const int64_t bt = pos[r] / B;
    for (int g = 0; g < hkv; ++g) {
      double* srow = S + (r * hkv + g) * nblk;
      for (int64_t j = 0; j < nblk; ++j) {
        if (j >= bt) { srow[j] = nan; continue; }
        double s = 0.0;
        for (int h = g * G; h < (g + 1) * G; ++h)
          for (int i = 0; i < d; ++i)
            s += elem(Q, dtype, (r * hq + h) * (int64_t)d + i) * C[(j * hkv + g) * (int64_t)d + i];
        srow[j] = s;
      }
    }
  }
}

// Exp-free top-k: the own block b = floor(pos/B) plus the best min(k-1, b)
// candidates under the order (score descending, block index ascending).
// idx[r][g][0..k) receives the chosen blocks in ascending order, padded with -1.
// gap[r][g] = (score of the last chosen candidate) - (score of the best
// rejected one), +inf when nothing is rejected (b <= k-1).
void orc_select(const double* S, int64_t R, const int64_t* pos, int hkv, int64_t nblk, int B,
                int k, int32_t* idx, double* gap) {
  const double inf = std::numeric_limits<double>::infinity();
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < R; ++r) {
    const int64_t bt = pos[r] / B;
    for (int g = 0; g < hkv; ++g) {
      const double* srow = S + (r * hkv + g) * nblk;
      std::vector<int64_t> cand;
      for (int64_t j = 0; j < bt; ++j) cand.push_back(j);
      std::sort(cand.begin(), cand.end(), [&](int64_t a, int64_t b) {
        if (srow[a] != srow[b]) return srow[a] > srow[b];
        return a < b;
      });
      const int64_t take = std::min<int64_t>(k - 1, bt);
      std::vector<int64_t> chosen(cand.begin(), cand.begin() + take);
      chosen.push_back(bt);
      std::sort(chosen.begin(), chosen.end());
      int32_t* out = idx + (r * hkv + g) * (int64_t)k;
      for (int s = 0; s < k; ++s) out[s] = s < (int)chosen.size() ? (int32_t)chosen[s] : -1;
      // k == 1 keeps only the own block whatever the scores: no decision, gap +inf
      gap[r * hkv + g] = (take > 0 && take < bt) ? srow[cand[take - 1]] - srow[cand[take]] : inf;
    }
  }
}

// Exact attention over the selected blocks. For row r, head h (group g):
// keys u of the listed blocks with u <= pos[r] and u < L; logits
// l_u = scale * q . k_u; w = softmax(l); O = sum_u w_u v_u; lse = log sum exp(l).
// idx entries < 0 are padding; entries may come in any order. The attended
// tokens form a set, so a block listed twice in a row counts once.
void orc_attend(const void* Q, const void* K, const void* V, int dtype, int64_t R,
                const int64_t* pos, int64_t L, int hq, int hkv, int d, int B, const int32_t* idx,
                int k, double scale, double* O, double* lse) {
  const int G = hq / hkv;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < R; ++r) {
    for (int h = 0; h < hq; ++h) {
      const int g = h / G;
      const int32_t* blocks = idx + (r * hkv + g) * (int64_t)k;
      std::vector<int64_t> keys_u;
      for (int s = 0; s < k; ++s) {
        if (blocks[s] < 0) continue;
        bool seen = false;
        for (int s2 = 0; s2 < s; ++s2) seen = seen || blocks[s2] == blocks[s];
        if (seen) continue;
        for (int64_t u = (int64_t)blocks[s] * B; u < (int64_t)(blocks[s] + 1) * B; ++u)
          if (u <= pos[r] && u < L) keys_u.push_back(u);
      }
      std::vector<double> logit(keys_u.size());
      double m = -std::numeric_limits<double>::infinity();
      for (size_t n = 0; n < keys_u.size(); ++n) {
        double s = 0.0;
        for (int i = 0; i < d; ++i)
          s += elem(Q, dtype, (r * hq + h) * (int64_t)d + i) *
               elem(K, dtype, (keys_u[n] * hkv + g) * (int64_t)d + i);
        logit[n] = s * scale;
        m = std::max(m, logit[n]);
      }
      double z = 0.0;
      for (size_t n = 0; n < keys_u.size(); ++n) z += std::exp(logit[n] - m);
      double* o = O + (r * hq + h) * (int64_t)d;
      for (int i = 0; i < d; ++i) o[i] = 0.0;
      for (size_t n = 0; n < keys_u.size(); ++n) {
        const double w = std::exp(logit[n] - m) / z;
        for (int i = 0; i < d; ++i) o[i] += w * elem(V, dtype, (keys_u[n] * hkv + g) * (int64_t)d + i);
      }
      lse[r * hq + h] = keys_u.empty() ? -std::numeric_limits<double>::infinity() : m + std::log(z);
    }
  }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
