// msa_topk_blocks: per (query row, KV group) causal top-k block selection.
//
// Rule (inteligile "MiniMax-M3" model page, "Checked in its code", row
// "Indexer-selected sparse attention": k = min(topk_blocks, #key blocks) and
// a -inf-scored slot is reported as -1; current-block forcing and the
// lower-id tie-break are this library's stated reading):
//   cur = p // block_size is always kept; the other topk-1 slots go to the
//   best earlier blocks b < cur with a finite score, ranked by
//   (score desc, b asc); ids are written ascending, padded with -1.
//
// "Exp-free": selection runs on the raw fp32 scores (softmax is monotone).
// Each candidate becomes a distinct 64-bit key (order-preserving score bits,
// then the complement of its block id); the answer is every key at or above
// the (topk-1)-th largest.  One warp per row (up to 1024 blocks) first finds
// the (topk-1)-th largest of its 32 lane maxima, a lower bound of that
// threshold, and ranks exactly the few keys at or above it.  Wider rows, and
// rows where that candidate set is large, run an MSB-first bitwise search
// whose counts are warp reductions (redux.sync), stopping as soon as exactly
// topk-1 keys lie above the probe.
#pragma once
#include "common.cuh"

namespace msa {

template <int W, int NPER>
__global__ void __launch_bounds__(W == 1 ? 128 : 32 * W)
topk_blocks_kernel(const float* __restrict__ scores, int32_t* __restrict__ out,
                   const int32_t* __restrict__ q_start, const int32_t* __restrict__ ctx_len, int num_seqs,
                   int total_q, int Hkv, int max_blocks, int topk, int block_size) {
  constexpr int THREADS = 32 * W;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  long row;                 // (t, g) row handled by this warp (W == 1) or CTA
  if (W == 1) row = static_cast<long>(blockIdx.x) * 4 + warp;
  else row = blockIdx.x;
  const long nrows = static_cast<long>(total_q) * Hkv;
  __shared__ int s_cnt[W > 1 ? W : 1];
  __shared__ int s_sel[W > 1 ? 64 : 1];
  __shared__ int s_nsel;
  __shared__ uint64_t s_cand[W == 1 ? 4 : 1][64];   // fast-path candidates, one area per warp
  __shared__ uint64_t s_thr[W == 1 ? 4 : 1];
  if (row >= nrows) return;  // W == 1: whole warp leaves together; W > 1: whole CTA
  const int tid = (W == 1) ? lane : static_cast<int>(threadIdx.x);
  const int t = static_cast<int>(row / Hkv);
  const int s = find_seq(q_start, num_seqs, t);
  const int qs = __ldg(q_start + s);
  const int nq = __ldg(q_start + s + 1) - qs;
  const long p = static_cast<long>(__ldg(ctx_len + s)) - nq + (t - qs);
  int32_t* orow = out + row * topk;
  if (p < 0 || p / block_size >= max_blocks) {
    if (tid == 0) flag_error(MSA_DEV_BOUNDS);
    for (int j = tid; j < topk; j += THREADS) orow[j] = -1;
    return;
  }
  const int cur = static_cast<int>(p / block_size);
  const float* srow = scores + row * static_cast<long>(max_blocks);

  // load candidates b < cur with a finite score.  Every lane issues all NPER
  // loads before using any (an in-bounds clamped address where b >= cur), so
  // they are in flight together instead of one round trip each.
  float sv[NPER];
  const int last = cur > 0 ? cur - 1 : 0;
#pragma unroll
  for (int i = 0; i < NPER; ++i) sv[i] = __ldcs(srow + min(tid + i * THREADS, last));
  uint64_t key[NPER];
  int nvalid = 0;
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int b = tid + i * THREADS;
    const bool ok = b < cur && sv[i] > -INFINITY;  // excludes -inf and NaN
    key[i] = ok ? (static_cast<uint64_t>(order_key(sv[i])) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - b) : 0ull;
    nvalid += ok ? 1 : 0;
  }
  auto block_sum = [&](int v) -> int {
    v = __reduce_add_sync(0xFFFFFFFFu, v);
    if (W == 1) return v;
    if (lane == 0) s_cnt[warp] = v;
    __syncthreads();
    int tot = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) tot += s_cnt[w];
    __syncthreads();
    return tot;
  };
  const int m = topk - 1;  // free slots besides the current block
  const int total_valid = block_sum(nvalid);
  const bool take_all = total_valid <= m;
  uint64_t thr = 1;  // keep valid keys >= thr
  bool found = false;
  if (W == 1 && !take_all && m > 0 && m <= 32) {
    // Fast path.  The m-th largest of the 32 lane maxima bounds the m-th
    // largest key from below (those m lane maxima are m distinct keys), so the
    // answer is among the few keys at or above it: rank those exactly.
    uint64_t lmax = 0;
#pragma unroll
    for (int i = 0; i < NPER; ++i) lmax = key[i] > lmax ? key[i] : lmax;
    uint64_t lo = 0;
    for (int bit = 63; bit >= 0; --bit) {
      const uint64_t probe = lo | (1ull << bit);
      const int c = __popc(__ballot_sync(0xFFFFFFFFu, lmax >= probe));
      if (c >= m) {
        lo = probe;
        if (c == m) break;
      }
    }
    if (lo != 0) {
      int cl = 0;
#pragma unroll
      for (int i = 0; i < NPER; ++i) cl += (key[i] >= lo) ? 1 : 0;
      int incl = cl;  // inclusive prefix over lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += n;
      }
      const int ncand = __shfl_sync(0xFFFFFFFFu, incl, 31);
      if (ncand <= 64) {
        uint64_t* cand = s_cand[warp];
        int at = incl - cl;
#pragma unroll
        for (int i = 0; i < NPER; ++i)
          if (key[i] >= lo) cand[at++] = key[i];
        __syncwarp();
        for (int c = lane; c < ncand; c += 32) {
          const uint64_t kc = cand[c];
          int above = 0;
          for (int d = 0; d < ncand; ++d) above += (cand[d] > kc) ? 1 : 0;
          if (above == m - 1) s_thr[warp] = kc;   // exactly one candidate: keys are distinct
        }
        __syncwarp();
        thr = s_thr[warp];
        found = true;
      }
    }
  }
  if (!take_all && m > 0 && !found) {
    uint64_t prefix = 0;
    for (int bit = 63; bit >= 0; --bit) {
      const uint64_t probe = prefix | (1ull << bit);
      int c = 0;
#pragma unroll
      for (int i = 0; i < NPER; ++i) c += (key[i] >= probe) ? 1 : 0;
      const int tot = block_sum(c);
      if (tot >= m) {
        prefix = probe;
        if (tot == m) break;  // keys are distinct: exactly the m best lie above
      }
    }
    thr = prefix;
  }
  // valid keys are distinct and non-zero; invalid ones are 0
  // write the selected ids ascending, then cur, then -1 padding
  if (W == 1) {
    int base = 0;
#pragma unroll
    for (int i = 0; i < NPER; ++i) {
      const bool sel = m > 0 && key[i] != 0 && key[i] >= thr;
      const unsigned msk = __ballot_sync(0xFFFFFFFFu, sel);
      if (sel) orow[base + __popc(msk & ((1u << lane) - 1u))] = tid + i * THREADS;
      base += __popc(msk);
    }
    for (int j = base + lane; j < topk; j += 32) orow[j] = (j == base) ? cur : -1;
  } else {
    if (threadIdx.x == 0) s_nsel = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < NPER; ++i) {
      if (m > 0 && key[i] != 0 && key[i] >= thr) {
        const int at = atomicAdd(&s_nsel, 1);
        if (at < 64) s_sel[at] = tid + i * THREADS;
      }
    }
    __syncthreads();
    const int n = min(s_nsel, 64);
    if (warp == 0) {
      // rank sort of <= 64 distinct ids
      for (int a = lane; a < n; a += 32) {
        const int v = s_sel[a];
        int rank = 0;
        for (int c = 0; c < n; ++c) rank += (s_sel[c] < v) ? 1 : 0;
        orow[rank] = v;
      }
      for (int j = n + lane; j < topk; j += 32) orow[j] = (j == n) ? cur : -1;
    }
  }
}

}  // namespace msa
