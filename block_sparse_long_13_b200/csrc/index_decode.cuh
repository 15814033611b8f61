// msa_index_scores, streaming form (few queries per sequence: decode and
// speculative verify).
//
// Computes, for every query row r of sequence s (position p_r), KV group g
// and block b of the sequence:
//   S_g(r, b) = sum_{h in heads(g)} max_{j in block b, j <= p_r} q_h(r) . k_h(j)
// (inteligile "MiniMax-M3" model page, row "Indexer-selected sparse
// attention": per-head key scores pooled into blocks; 24-ai.news, every
// query group scores all available 128-token blocks).  Pooling = max and the
// sum over a group's indexer heads are this library's stated reading.
//
// The pass is HBM-bound: every indexer key of every visible page is read
// once.  Persistent CTAs (one per SM) own contiguous runs of (sequence,
// page) units; each unit is read as H_kv TMA tiles of hg x 128 x 64 bf16
// (hg = indexer heads per group, 128-byte swizzle) through a STAGES-deep
// ring of shared-memory buffers.  Each thread owns one key row, widens it to
// fp32 and dots it with the sequence's (<= 8) queries held in shared memory;
// the block max is a warp redux.sync on order-preserving integer keys.
#pragma once
#include "common.cuh"

namespace msa {

constexpr int IDXD_THREADS = 256;
constexpr int IDXD_MAXQ = 8;       // queries per sequence handled by this form
constexpr int IDXD_MAXHG = 8;      // indexer heads per KV group
constexpr int IDXD_MAXHI = 16;     // indexer heads
constexpr int IDXD_MAXSEQ = 2048;  // sequences per call for this form
constexpr int IDXD_RING_BYTES = 160 * 1024;

struct IdxDecodeArgs {
  const __nv_bfloat16* idx_q;   // [total_q][Hi][64]
  float* scores;                // [total_q][Hkv][max_blocks]
  const int32_t* q_start;
  const int32_t* ctx_len;
  const int32_t* page_table;    // [num_seqs][max_blocks]
  int num_seqs, max_blocks, num_pages, Hi, Hkv, hg, block_size;
  int stage_bytes, stages;
};

__global__ void __launch_bounds__(IDXD_THREADS, 1)
index_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, const IdxDecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full_bar[16];
  __shared__ int s_nbprefix[IDXD_MAXSEQ + 1];
  __shared__ __align__(16) float s_q[IDXD_MAXQ * IDXD_MAXHI * 64];  // current sequence: queries of all heads (fp32)
  __shared__ uint32_t s_part[2][IDXD_MAXQ][IDXD_MAXHG][4];
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int token = tid & 127;
  const int hl0 = tid >> 7;  // 0 or 1

  // blocks per sequence (0 for sequences without queries), prefix in smem
  if (tid == 0) {
    s_abort = 0;
    int acc = 0;
    s_nbprefix[0] = 0;
    for (int s = 0; s < a.num_seqs; ++s) {
      const int nq = __ldg(a.q_start + s + 1) - __ldg(a.q_start + s);
      int nb = (__ldg(a.ctx_len + s) + a.block_size - 1) / a.block_size;
      if (nq <= 0) nb = 0;
      nb = min(nb, a.max_blocks);
      acc += nb;
      s_nbprefix[s + 1] = acc;
    }
    for (int i = 0; i < a.stages; ++i) mbar_init(&full_bar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const long total_units = s_nbprefix[a.num_seqs];
  const long u0 = total_units * blockIdx.x / gridDim.x;
  const long u1 = total_units * (blockIdx.x + 1) / gridDim.x;
  const long nstage = (u1 - u0) * a.Hkv;
  if (nstage == 0) return;

  // unit -> (seq, block): seq-major walk
  auto locate = [&](long u, int& s, int& b) {
    int lo = 0, hi = a.num_seqs - 1;
    while (lo < hi) {  // largest s with prefix[s] <= u
      const int mid = (lo + hi + 1) >> 1;
      if (s_nbprefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    s = lo;
    b = static_cast<int>(u - s_nbprefix[lo]);
  };

  // producer state (thread 0): issue stage k into slot k % stages
  auto issue = [&](long k) {
    const long u = u0 + k / a.Hkv;
    const int g = static_cast<int>(k % a.Hkv);
    int s, b;
    locate(u, s, b);
    int page = __ldg(a.page_table + static_cast<long>(s) * a.max_blocks + b);
    if (page < 0 || page >= a.num_pages) { flag_error(MSA_DEV_BOUNDS); page = 0; }
    const int slot = static_cast<int>(k % a.stages);
    mbar_arrive_expect_tx(&full_bar[slot], a.stage_bytes);
    tma_load_4d(ring + static_cast<long>(slot) * a.stage_bytes, &tmap_k, &full_bar[slot], 0, 0, g * a.hg, page);
  };
  long issued = 0, kstop = -1;
  if (tid == 0) {
    tma_prefetch_desc(&tmap_k);
    for (long k = 0; k < nstage && k < a.stages; ++k) { issue(k); ++issued; }
  }

  int cur_seq = -1, nq = 0, qrow0 = 0, ctx = 0;
  for (long k = 0; k < nstage; ++k) {
    const long u = u0 + k / a.Hkv;
    const int g = static_cast<int>(k % a.Hkv);
    int s, b;
    locate(u, s, b);
    if (s != cur_seq) {
      // load this sequence's queries (all indexer heads) as fp32
      __syncthreads();
      cur_seq = s;
      qrow0 = __ldg(a.q_start + s);
      nq = __ldg(a.q_start + s + 1) - qrow0;
      ctx = __ldg(a.ctx_len + s);
      if (nq > IDXD_MAXQ) { if (tid == 0) flag_error(MSA_DEV_BOUNDS); nq = IDXD_MAXQ; }
      const int n = nq * a.Hi * 64;
      const __nv_bfloat16* src = a.idx_q + static_cast<long>(qrow0) * a.Hi * 64;
      for (int i = tid; i < n; i += IDXD_THREADS) s_q[i] = __bfloat162float(src[i]);
      __syncthreads();
    }
    const int slot = static_cast<int>(k % a.stages);
    const uint32_t parity = static_cast<uint32_t>((k / a.stages) & 1);
    const bool ok = mbar_wait(&full_bar[slot], parity, &s_abort);
    const uint8_t* tile = ring + static_cast<long>(slot) * a.stage_bytes;
    const int j = b * a.block_size + token;  // absolute key position
    const int pbuf = static_cast<int>(k & 1);
    for (int hl = hl0; ok && hl < a.hg; hl += 2) {
      // this thread's key row: 64 bf16, 128-byte swizzled
      const uint8_t* rowp = tile + (hl * 128 + token) * 128;
      float acc[IDXD_MAXQ];
#pragma unroll
      for (int i = 0; i < IDXD_MAXQ; ++i) acc[i] = 0.f;
      const int h = g * a.hg + hl;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((c ^ (token & 7)) << 4));
        const float kf[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                             bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
        for (int i = 0; i < IDXD_MAXQ; ++i) {
          if (i < nq) {
            const float4* qp = reinterpret_cast<const float4*>(s_q + (i * a.Hi + h) * 64 + c * 8);
            const float4 q0 = qp[0], q1 = qp[1];
            float t = acc[i];
            t = fmaf(q0.x, kf[0], t); t = fmaf(q0.y, kf[1], t); t = fmaf(q0.z, kf[2], t); t = fmaf(q0.w, kf[3], t);
            t = fmaf(q1.x, kf[4], t); t = fmaf(q1.y, kf[5], t); t = fmaf(q1.z, kf[6], t); t = fmaf(q1.w, kf[7], t);
            acc[i] = t;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < IDXD_MAXQ; ++i) {
        if (i < nq) {
          const int p = ctx - nq + i;
          const float v = (j <= p) ? acc[i] : -INFINITY;
          const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, order_key(v));
          if (lane == 0) s_part[pbuf][i][hl][warp & 3] = m;
        }
      }
    }
    __syncthreads();  // slot consumed, partial maxima visible, abort flag uniform
    if (s_abort) { kstop = k; break; }
    if (tid == 0 && k + a.stages < nstage) { issue(k + a.stages); ++issued; }
    if (tid < nq) {
      float tot = 0.f;
      for (int hl = 0; hl < a.hg; ++hl) {
        const uint32_t* pp = s_part[pbuf][tid][hl];
        const uint32_t m = max(max(pp[0], pp[1]), max(pp[2], pp[3]));
        tot += key_to_float(m);
      }
      a.scores[(static_cast<long>(qrow0 + tid) * a.Hkv + g) * a.max_blocks + b] = tot;
    }
  }
  // after a timeout, let the copies still in flight land (bounded) before the CTA exits
  if (tid == 0 && kstop >= 0) {
    for (long kk = kstop; kk < issued; ++kk)
      mbar_wait_drain(&full_bar[kk % a.stages], static_cast<uint32_t>((kk / a.stages) & 1));
  }
}

}  // namespace msa
