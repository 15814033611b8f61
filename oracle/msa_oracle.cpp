// Plain CPU oracle for the MiniMax Sparse Attention (MSA) hot path, in C++.
//
// TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
// the benchmark's CPU-baseline / reference arm may load this library.  It
// shares no code with the CUDA library (no header, helper or table) and
// includes nothing from it.
//
// Every value is computed in double, one definition at a time, in the order the
// method states them; results are returned in double.  Sources (page title,
// then section):
//
// * [daily.dev] "MiniMax M3: 1M-token multimodal reasoning model now available
//   with NVIDIA and vLLM support", sections "Summary" and "What makes M3
//   different": the KV sequence is cut into 128-token blocks, every block is
//   scored, and only the top blocks are attended per query.
// * [inteligile] "MiniMax-M3" model page, table "Checked in its code":
//   row "Indexer-selected sparse attention" (per-head key scores pooled into
//   blocks; k = min(topk_blocks, number of key blocks) kept per query; a kept
//   slot whose score is -inf reported as -1); row "Grouped-query attention"
//   (query head h reads KV head h / (H_q / H_kv)); rows "Learnable attention
//   sink" and "Gated attention output" (plain softmax: no sink logit, no gate);
//   tags "Two-phase forward", "LSE fusion".
// * [24-ai.news] "MiniMax M3 in vLLM: Day-0-Unterstuetzung ...", section "Warum
//   ist ein Million-Token-Kontext eine Serving-Herausforderung?": each query or
//   GQA query group scores every available 128-token block with light indexer
//   kernels and keeps the most relevant ones.
//
// Readings where the pages leave a step open: pooling = max over the block's
// causally visible keys (j <= p); the indexer heads are split contiguously over
// the KV groups and a group's block score is the SUM of its heads' pooled
// scores; raw dot products; the query's own block cur = p / block_size always
// takes one of the k slots, the other k-1 go to the best earlier blocks by
// (score descending, block ascending); softmax scale 1/sqrt(head_dim) unless
// given; selected ids ascending, padded with -1.
//
// Threads (std::thread) split the independent outputs of a call -- (row,
// block) score entries, (row, group) attention results -- into contiguous
// ranges; every output is computed by one thread from the definition alone, so
// the results do not depend on the thread count.
//
// Parity pins: tests/test_oracle_pins.py runs every pin against this library
// and against the float64 numpy oracle, and tests/test_oracle_cpp.py checks the
// two against each other.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <limits>
#include <thread>
#include <vector>

namespace {

const double kNegInf = -std::numeric_limits<double>::infinity();

// Run body(i) for i in [0, n) on up to `threads` threads, contiguous ranges.
template <class F>
void parallel_for(int64_t n, int threads, F body) {
  if (threads <= 0) threads = static_cast<int>(std::max(1u, std::thread::hardware_concurrency()));
  if (n <= 0) return;
  const int64_t t = std::min<int64_t>(threads, n);
  if (t <= 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(static_cast<size_t>(t));
  for (int64_t w = 0; w < t; ++w) {
    const int64_t lo = n * w / t, hi = n * (w + 1) / t;
    pool.emplace_back([lo, hi, &body] {
      for (int64_t i = lo; i < hi; ++i) body(i);
    });
  }
  for (auto& th : pool) th.join();
}

// 1. Indexer block scores.  For row r at position p, KV group g and block b:
//   S_g(r, b) = sum over h in heads(g) of  max over keys j of block b with j <= p of  q_h(r) . k_h(j),
// heads(g) = {g*Hi/Hkv, ..., (g+1)*Hi/Hkv - 1}; a block with no visible key scores -inf.
template <class T>
void block_scores(const T* idx_q, const int64_t* pos, int64_t n, int Hi, int di, const T* idx_k, int64_t L,
                  int Hkv, int bs, int nb_out, double* out, int threads) {
  const int per = Hi / Hkv;
  parallel_for(n * nb_out, threads, [&](int64_t item) {
    const int64_t r = item / nb_out;
    const int b = static_cast<int>(item % nb_out);
    const int64_t p = pos[r];
    const int64_t lo = static_cast<int64_t>(b) * bs;
    const int64_t hi = std::min<int64_t>(lo + bs, L);   // keys of block b that exist
    for (int g = 0; g < Hkv; ++g) out[(r * Hkv + g) * nb_out + b] = kNegInf;
    if (lo > p || lo >= hi) return;                      // no visible key in this block
    for (int g = 0; g < Hkv; ++g) {
      double sum = 0.0;
      for (int h = g * per; h < (g + 1) * per; ++h) {
        double best = kNegInf;
        for (int64_t j = lo; j < hi && j <= p; ++j) {
          double dot = 0.0;
          for (int c = 0; c < di; ++c)
            dot += static_cast<double>(idx_q[(r * Hi + h) * di + c]) * static_cast<double>(idx_k[(j * Hi + h) * di + c]);
          best = std::max(best, dot);
        }
        sum += best;
      }
      out[(r * Hkv + g) * nb_out + b] = sum;
    }
  });
}

// Ranked candidates of one row: earlier blocks b < cur (and < nb) whose score is not -inf,
// ordered by (score descending, block ascending).
std::vector<int> ranked_candidates(const double* row, int64_t cur, int nb) {
  std::vector<int> cand;
  const int64_t upto = std::min<int64_t>(cur, nb);
  for (int b = 0; b < upto; ++b)
    if (row[b] != kNegInf) cand.push_back(b);
  std::sort(cand.begin(), cand.end(), [row](int a, int c) {
    if (row[a] != row[c]) return row[a] > row[c];
    return a < c;
  });
  return cand;
}

// 3. Sparse GQA attention over the selected blocks.  Query head h of row r (group
// g = h / (Hq/Hkv)) reads the keys j <= p of the blocks in sel[r][g][:]; with
// s_j = scale * q_h . k_j and m = max_j s_j:  out = sum_j e^{s_j - m} v_j / sum_j e^{s_j - m},
// lse = m + log sum_j e^{s_j - m}.  A (row, group) with no key gets out = 0, lse = -inf.
template <class T>
void sparse_attention(const T* q, const int64_t* pos, int64_t n, int Hq, int d, const T* const* kblk,
                      const T* const* vblk, const int32_t* blk_len, int64_t nblk, int Hkv, const int32_t* sel,
                      int topk, int bs, double scale, double* out, double* lse, int threads, int* bad) {
  const int G = Hq / Hkv;
  parallel_for(n * Hkv, threads, [&](int64_t item) {
    const int64_t r = item / Hkv;
    const int g = static_cast<int>(item % Hkv);
    const int64_t p = pos[r];
    // the keys this (row, group) sees: (block, row inside the block), in slot order
    std::vector<std::pair<int64_t, int>> keys;
    for (int s = 0; s < topk; ++s) {
      const int64_t b = sel[(r * Hkv + g) * topk + s];
      if (b < 0) continue;
      if (b >= nblk || kblk[b] == nullptr || vblk[b] == nullptr) {
        *bad = 1;
        continue;
      }
      for (int i = 0; i < blk_len[b]; ++i)
        if (b * bs + i <= p) keys.emplace_back(b, i);
    }
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      double* o = out + (r * Hq + h) * d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      if (keys.empty()) {
        lse[r * Hq + h] = kNegInf;
        continue;
      }
      std::vector<double> s(keys.size());
      double m = kNegInf;
      for (size_t k = 0; k < keys.size(); ++k) {
        const T* kr = kblk[keys[k].first] + (static_cast<int64_t>(keys[k].second) * Hkv + g) * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += static_cast<double>(q[(r * Hq + h) * d + c]) * static_cast<double>(kr[c]);
        s[k] = scale * dot;
        m = std::max(m, s[k]);
      }
      double l = 0.0;
      for (size_t k = 0; k < keys.size(); ++k) {
        const double e = std::exp(s[k] - m);
        l += e;
        const T* vr = vblk[keys[k].first] + (static_cast<int64_t>(keys[k].second) * Hkv + g) * d;
        for (int c = 0; c < d; ++c) o[c] += e * static_cast<double>(vr[c]);
      }
      for (int c = 0; c < d; ++c) o[c] /= l;
      lse[r * Hq + h] = m + std::log(l);
    }
  });
}

}  // namespace

extern "C" {

int oracle_hardware_threads(void) { return static_cast<int>(std::thread::hardware_concurrency()); }

int oracle_block_scores_f32(const float* idx_q, const int64_t* pos, int64_t n, int Hi, int di, const float* idx_k,
                            int64_t L, int Hkv, int bs, int nb_out, double* out, int threads) {
  if (Hkv <= 0 || Hi % Hkv != 0 || bs <= 0) return 1;
  block_scores(idx_q, pos, n, Hi, di, idx_k, L, Hkv, bs, nb_out, out, threads);
  return 0;
}

int oracle_block_scores_f64(const double* idx_q, const int64_t* pos, int64_t n, int Hi, int di, const double* idx_k,
                            int64_t L, int Hkv, int bs, int nb_out, double* out, int threads) {
  if (Hkv <= 0 || Hi % Hkv != 0 || bs <= 0) return 1;
  block_scores(idx_q, pos, n, Hi, di, idx_k, L, Hkv, bs, nb_out, out, threads);
  return 0;
}

// 2. Top-k selection.  R = {cur} U the min(topk-1, #candidates) best candidates, written
// ascending and padded with -1 to topk entries (-inf scores are never kept).  The comparisons
// are made on the values given (callers pass fp32 scores widened exactly, as the kernel sees them).
int oracle_select_blocks(const double* scores, const int64_t* pos, int64_t n, int G, int nb, int topk, int bs,
                         int32_t* out) {
  if (topk <= 0 || bs <= 0) return 1;
  for (int64_t r = 0; r < n; ++r) {
    const int64_t cur = pos[r] / bs;
    for (int g = 0; g < G; ++g) {
      const std::vector<int> ranked = ranked_candidates(scores + (r * G + g) * nb, cur, nb);
      std::vector<int64_t> chosen(ranked.begin(), ranked.begin() + std::min<size_t>(ranked.size(), topk - 1));
      chosen.push_back(cur);
      std::sort(chosen.begin(), chosen.end());
      int32_t* o = out + (r * G + g) * topk;
      for (int s = 0; s < topk; ++s) o[s] = s < static_cast<int>(chosen.size()) ? static_cast<int32_t>(chosen[s]) : -1;
    }
  }
  return 0;
}

// Near-tie report of the selection boundary: s_a is the (topk-1)-th ranked candidate score (the
// last one kept), s_b the next one; near when |s_a - s_b| < 1e-3 * max(|s_a|, 1e-6).  Rows with
// no rejected candidate are never near-ties (s_a = s_b = NaN there).
int oracle_boundary_gap(const double* scores, const int64_t* pos, int64_t n, int G, int nb, int topk, int bs,
                        uint8_t* near, double* sa, double* sb) {
  if (bs <= 0) return 1;
  const int m = topk - 1;
  for (int64_t r = 0; r < n; ++r) {
    const int64_t cur = pos[r] / bs;
    for (int g = 0; g < G; ++g) {
      const double* row = scores + (r * G + g) * nb;
      const std::vector<int> ranked = ranked_candidates(row, cur, nb);
      const int64_t i = r * G + g;
      near[i] = 0;
      sa[i] = sb[i] = std::numeric_limits<double>::quiet_NaN();
      if (m < 1 || static_cast<int>(ranked.size()) <= m) continue;
      const double a = row[ranked[m - 1]], b = row[ranked[m]];
      sa[i] = a;
      sb[i] = b;
      near[i] = std::fabs(a - b) < 1e-3 * std::max(std::fabs(a), 1e-6) ? 1 : 0;
    }
  }
  return 0;
}

int oracle_sparse_attention_f32(const float* q, const int64_t* pos, int64_t n, int Hq, int d, const float* const* kblk,
                                const float* const* vblk, const int32_t* blk_len, int64_t nblk, int Hkv,
                                const int32_t* sel, int topk, int bs, double scale, double* out, double* lse,
                                int threads) {
  if (Hkv <= 0 || Hq % Hkv != 0) return 1;
  int bad = 0;
  sparse_attention(q, pos, n, Hq, d, kblk, vblk, blk_len, nblk, Hkv, sel, topk, bs, scale, out, lse, threads, &bad);
  return bad ? 2 : 0;
}

int oracle_sparse_attention_f64(const double* q, const int64_t* pos, int64_t n, int Hq, int d,
                                const double* const* kblk, const double* const* vblk, const int32_t* blk_len,
                                int64_t nblk, int Hkv, const int32_t* sel, int topk, int bs, double scale, double* out,
                                double* lse, int threads) {
  if (Hkv <= 0 || Hq % Hkv != 0) return 1;
  int bad = 0;
  sparse_attention(q, pos, n, Hq, d, kblk, vblk, blk_len, nblk, Hkv, sel, topk, bs, scale, out, lse, threads, &bad);
  return bad ? 2 : 0;
}

// 4. Two-phase forward: S partial attentions over disjoint key sets, each normalised over its own
// keys, combined by their log-sum-exp:  L = log sum_s e^{lse_s},  out = sum_s e^{lse_s - L} out_s.
// Partials with lse = -inf weigh nothing; a unit whose partials are all -inf gets out = 0, L = -inf.
int oracle_merge_partials(const double* outs, const double* lses, int S, int64_t units, int d, double* out,
                          double* lse) {
  for (int64_t u = 0; u < units; ++u) {
    double mx = kNegInf;
    for (int s = 0; s < S; ++s) mx = std::max(mx, lses[s * units + u]);
    double* o = out + u * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (mx == kNegInf) {
      lse[u] = kNegInf;
      continue;
    }
    double tot = 0.0;
    for (int s = 0; s < S; ++s) tot += std::exp(lses[s * units + u] - mx);
    const double L = mx + std::log(tot);
    for (int s = 0; s < S; ++s) {
      const double w = std::exp(lses[s * units + u] - L);
      for (int c = 0; c < d; ++c) o[c] += w * outs[(s * units + u) * d + c];
    }
    lse[u] = L;
  }
  return 0;
}

}  // extern "C"
