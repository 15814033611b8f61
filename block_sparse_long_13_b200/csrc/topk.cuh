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
  if (!take_all && m > 0) {
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


// One warp per (row, group) for rows of up to 32 * NPER candidates.  Scores are
// compared as 32-bit order-preserving keys; ties are broken by the lower block
// id only where they matter.  The (topk-1)-th largest of the 32 lane maxima
// bounds the threshold from below, so the answer lies among the few candidates
// at or above it; those are ranked exactly, and the selected ids are sorted by
// id for the output.  Rows where that set is large (or topk-1 > 32) take the
// MSB-first bitwise search on 64-bit keys.  Eight 4-warp CTAs per SM (64
// registers): the per-row search and ranking are latency chains, so residency
// pays (-11 % against five CTAs per SM at 96 registers).
template <int NPER>
__global__ void __launch_bounds__(128, 8) topk_row_warp_kernel(const float* __restrict__ scores, int32_t* __restrict__ out,
                                                            const int32_t* __restrict__ q_start,
                                                            const int32_t* __restrict__ ctx_len, int num_seqs,
                                                            int total_q, int Hkv, int max_blocks, int topk,
                                                            int block_size) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long row = static_cast<long>(blockIdx.x) * 4 + warp;
  __shared__ uint32_t s_ck[4][64];
  __shared__ int s_cb[4][64];
  __shared__ int s_sel[4][64];
  if (row >= static_cast<long>(total_q) * Hkv) return;   // whole warp
  const int t = static_cast<int>(row / Hkv);
  const int s = find_seq(q_start, num_seqs, t);
  const int qs = __ldg(q_start + s);
  const int nq = __ldg(q_start + s + 1) - qs;
  const long p = static_cast<long>(__ldg(ctx_len + s)) - nq + (t - qs);
  int32_t* orow = out + row * topk;
  if (p < 0 || p / block_size >= max_blocks) {
    if (lane == 0) flag_error(MSA_DEV_BOUNDS);
    for (int j = lane; j < topk; j += 32) orow[j] = -1;
    return;
  }
  const int cur = static_cast<int>(p / block_size);
  const float* srow = scores + row * static_cast<long>(max_blocks);
  // every load issued before any use (clamped in-bounds address where b >= cur)
  float sv[NPER];
  const int last = cur > 0 ? cur - 1 : 0;
#pragma unroll
  for (int i = 0; i < NPER; ++i) sv[i] = __ldcs(srow + min(lane + i * 32, last));
  uint32_t sk[NPER];   // order key of a finite candidate score (> 0), 0 otherwise
  int nvalid = 0;
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const bool ok = lane + i * 32 < cur && sv[i] > -INFINITY;   // excludes -inf and NaN
    sk[i] = ok ? order_key(sv[i]) : 0u;
    nvalid += ok ? 1 : 0;
  }
  const int m = topk - 1;   // free slots besides the current block
  const int total = __reduce_add_sync(0xFFFFFFFFu, nvalid);
  bool done = false;
  if (total > m && m > 0 && m <= 32) {
    uint32_t lmax = 0;
#pragma unroll
    for (int i = 0; i < NPER; ++i) lmax = max(lmax, sk[i]);
    uint32_t lo = 0;   // count(lane maxima >= lo) >= m
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t probe = lo | (1u << bit);
      const int c = __popc(__ballot_sync(0xFFFFFFFFu, lmax >= probe));
      if (c >= m) {
        lo = probe;
        if (c == m) break;
      }
    }
    if (lo != 0) {
      int cl = 0;
#pragma unroll
      for (int i = 0; i < NPER; ++i) cl += sk[i] >= lo ? 1 : 0;
      int incl = cl;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += n;
      }
      const int ncand = __shfl_sync(0xFFFFFFFFu, incl, 31);
      if (ncand <= 64) {
        int at = incl - cl;
#pragma unroll
        for (int i = 0; i < NPER; ++i) {
          if (sk[i] >= lo) {
            s_ck[warp][at] = sk[i];
            s_cb[warp][at] = lane + i * 32;
            ++at;
          }
        }
        __syncwarp();
        // rank by (score desc, id asc); the first m are the selection
        for (int c = lane; c < ncand; c += 32) {
          const uint32_t kc = s_ck[warp][c];
          const int bc = s_cb[warp][c];
          int rank = 0;
          for (int d = 0; d < ncand; ++d) {
            const uint32_t kd = s_ck[warp][d];
            rank += (kd > kc || (kd == kc && s_cb[warp][d] < bc)) ? 1 : 0;
          }
          if (rank < m) s_sel[warp][rank] = bc;
        }
        __syncwarp();
        // ids ascending, then the row's own block (every candidate lies before it)
        for (int j = lane; j < m; j += 32) {
          const int b = s_sel[warp][j];
          int r = 0;
          for (int k = 0; k < m; ++k) r += s_sel[warp][k] < b ? 1 : 0;
          orow[r] = b;
        }
        if (lane == 0) orow[m] = cur;
        done = true;
      }
    }
  }
  if (done) return;
  // general case: keep every candidate at or above the (m-th largest) 64-bit key
  uint64_t thr = 1;
  if (total > m && m > 0) {
    uint64_t prefix = 0;
    for (int bit = 63; bit >= 0; --bit) {
      const uint64_t probe = prefix | (1ull << bit);
      int c = 0;
#pragma unroll
      for (int i = 0; i < NPER; ++i) {
        const uint64_t key = sk[i] ? (static_cast<uint64_t>(sk[i]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(lane + i * 32)) : 0ull;
        c += key >= probe ? 1 : 0;
      }
      const int tot = __reduce_add_sync(0xFFFFFFFFu, c);
      if (tot >= m) {
        prefix = probe;
        if (tot == m) break;   // keys are distinct
      }
    }
    thr = prefix;
  }
  int base = 0;
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const uint64_t key = sk[i] ? (static_cast<uint64_t>(sk[i]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(lane + i * 32)) : 0ull;
    const bool sel = m > 0 && key != 0 && key >= thr;
    const unsigned msk = __ballot_sync(0xFFFFFFFFu, sel);
    if (sel) orow[base + __popc(msk & ((1u << lane) - 1u))] = lane + i * 32;
    base += __popc(msk);
  }
  for (int j = base + lane; j < topk; j += 32) orow[j] = (j == base) ? cur : -1;
}

}  // namespace msa
