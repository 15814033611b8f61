// msa_index_scores, streaming form on the tensor cores, for 3 to 16 queries per
// sequence (speculative verify and similar).
//
// Same definition as the other forms:
//   S_g(r, b) = sum_{h in heads(g)} max_{j in block b, j <= p_r} q_h(r) . k_h(j)
// (inteligile "MiniMax-M3" model page, row "Indexer-selected sparse
// attention"; 24-ai.news, every query group scores all available blocks).
//
// The CUDA-core streaming kernel reads each query value from shared memory
// once per key and query, so with several queries per sequence its
// shared-memory traffic, not HBM, sets the pace.  Here the products are one
// swap-AB tensor-core MMA per (block, head): D = K_h(b) Q_h^T with M = 128
// keys, N = 16 query rows of the sequence (the sequence's queries; the rest of
// the 16 rows are ignored), K = 64, the key tile straight from its TMA stage and
// the sequence's queries as a 16-row K-major tile per head.  Thread = key row
// reads its <= 16 scores from TMEM, masks keys after each query's position, and
// the block maximum is a warp redux on order-preserving integer keys plus a
// 4-warp exchange; the sum over the group's heads follows.
//
// Persistent CTAs (one per SM) own contiguous runs of (sequence, block) units
// as in the CUDA-core form; warp 0 streams the key tiles (and, when the
// sequence changes, its query tile), warp 1 issues the MMAs into a ring of TMEM
// accumulators, and two pooling groups (warps 2-5 and 6-9) take alternate
// stages: one group's per-stage chain (TMEM read, warp maxima, the previous
// stage's sums) is longer than the stream's time per stage.  Every wait is
// bounded.
#pragma once
#include "common.cuh"
#include "index_decode.cuh"

namespace msa {

constexpr int IDXT_GROUPS = 2;      // pooling groups of 4 warps, alternate stages
constexpr int IDXT_THREADS = 64 + IDXT_GROUPS * 128;
constexpr int IDXT_MAXHG = 4;       // indexer heads per KV group (the configuration allows at most 4)
constexpr int IDXT_MAXQ = 16;       // query rows per sequence (the MMA's N)
constexpr int IDXT_QHEAD = 2048;    // one head's query tile: 16 rows x 64 dims bf16, 128-byte swizzle

template <int NQ>
__global__ void __launch_bounds__(IDXT_THREADS, 1)
index_decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,   // keys (64, 128, Hi, P), box (64, 128, hg, 1)
                       const __grid_constant__ CUtensorMap tmap_q,   // idx_q (64, Hi, total_q), box (64, 1, 16)
                       const IdxDecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;                                            // a.stages x stage_bytes
  uint8_t* q_s = ring + static_cast<long>(a.stages) * a.stage_bytes;   // 2 x Hi x 2 KiB
  const int q_bytes = a.Hi * IDXT_QHEAD;
  __shared__ uint64_t full_bar[16], empty_bar[16], acc_full[8], acc_empty[8], q_full[2], q_empty[2], drain_bar;
  __shared__ int s_nbprefix[IDXD_MAXSEQ + 1];
  __shared__ uint32_t s_part[2 * IDXT_GROUPS][NQ][IDXT_MAXHG][4];   // per group, this and the previous stage
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nslot = min(8, 512 / (a.hg * 16));                    // TMEM accumulators in flight

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
    for (int i = 0; i < a.stages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 8; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(&drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const long total_units = s_nbprefix[a.num_seqs];
  const long u0 = total_units * blockIdx.x / gridDim.x;
  const long u1 = total_units * (blockIdx.x + 1) / gridDim.x;
  const long nstage = (u1 - u0) * a.Hkv;

  // unit -> (seq, block): seq-major order
  auto locate = [&](long u, int& s, int& b) {
    int lo = 0, hi = a.num_seqs - 1;
    while (lo < hi) {  // largest s with prefix[s] <= u
      const int mid = (lo + hi + 1) >> 1;
      if (s_nbprefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    s = lo;
    b = static_cast<int>(u - s_nbprefix[lo]);
  };
  // walking the units in order: (s, b) of the next unit
  auto advance = [&](int& s, int& b) {
    ++b;
    while (b >= s_nbprefix[s + 1] - s_nbprefix[s]) { ++s; b = 0; }
  };

  if (nstage > 0 && warp == 0) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_q);
    }
    int page_l = 0, seq_l = 0;
    int cur_seq = -1, nseq = 0;
    uint32_t used = 0, parity_bits = 0;   // per ring slot: issued at least once / parity of the last issue
    bool ok = true;
    // stage k = (unit j, group g) and its ring slot, kept as counters (no 64-bit division per stage)
    long j = 0;
    int g = 0, slot = 0;
    uint32_t par = 0;
    for (long k = 0; k < nstage && ok; ++k) {
      if (k > 0) {
        if (++g == a.Hkv) { g = 0; ++j; }
        if (++slot == a.stages) { slot = 0; par ^= 1u; }
      }
      if (g == 0 && (j & 31) == 0) {      // page ids (and sequences) of the next 32 units, one per lane
        const long uu = u0 + j + lane;
        page_l = 0;
        seq_l = 0;
        if (uu < u1) {
          int s, b;
          locate(uu, s, b);
          seq_l = s;
          page_l = __ldg(a.page_table + static_cast<long>(s) * a.max_blocks + b);
          if (page_l < 0 || page_l >= a.num_pages) { flag_error(MSA_DEV_BOUNDS); page_l = 0; }
        }
      }
      const int page = __shfl_sync(0xFFFFFFFFu, page_l, static_cast<int>(j & 31));
      const int seq = __shfl_sync(0xFFFFFFFFu, seq_l, static_cast<int>(j & 31));
      if (lane == 0) {
        if (seq != cur_seq) {             // the sequence's query tile: every indexer head's 16 rows
          const int qb = nseq & 1;
          ok = mbar_wait(&q_empty[qb], ((nseq >> 1) & 1) ^ 1, &s_abort);
          if (ok) {
            mbar_arrive_expect_tx(&q_full[qb], q_bytes);
            const int row0 = __ldg(a.q_start + seq);
            for (int h = 0; h < a.Hi; ++h)
              tma_load_3d(q_s + qb * q_bytes + h * IDXT_QHEAD, &tmap_q, &q_full[qb], 0, h, row0);
          }
          cur_seq = seq;
          ++nseq;
        }
        if (ok) ok = mbar_wait(&empty_bar[slot], par ^ 1u, &s_abort);
        if (ok) {
          mbar_arrive_expect_tx(&full_bar[slot], a.stage_bytes);
          tma_load_4d(ring + static_cast<long>(slot) * a.stage_bytes, &tmap_k, &full_bar[slot], 0, 0, g * a.hg, page);
          used |= 1u << slot;
          parity_bits = (parity_bits & ~(1u << slot)) | (par << slot);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && s_abort) {  // let issued copies land before the CTA exits
      for (int i = 0; i < a.stages; ++i)
        if (used & (1u << i)) mbar_wait_drain(&full_bar[i], (parity_bits >> i) & 1u);
      for (int b = 0; b < 2 && b < nseq; ++b) mbar_wait_drain(&q_full[b], (((nseq - 1 - b) >> 1) & 1));
    }
  } else if (nstage > 0 && warp == 1 && lane == 0) {
    // ------------------------------------------------------------ UMMA issuer
    const uint32_t idesc = idesc_bf16(128, 16, false, false);
    const uint64_t kdesc0 = sdesc_sw128(smem_u32(ring), 16, 1024);
    const uint64_t qdesc0 = sdesc_sw128(smem_u32(q_s), 16, 1024);
    int s, b;
    locate(u0, s, b);
    int cur_seq = -1, nseq = 0;
    bool ok = true;
    int g = 0, slot = 0, as = 0;
    uint32_t par = 0, apar = 0;
    for (long k = 0; k < nstage && ok && !s_abort; ++k) {
      if (k > 0) {
        if (++g == a.Hkv) { g = 0; advance(s, b); }
        if (++slot == a.stages) { slot = 0; par ^= 1u; }
        if (++as == nslot) { as = 0; apar ^= 1u; }
      }
      if (s != cur_seq) {
        if (cur_seq >= 0) umma_commit(&q_empty[(nseq - 1) & 1]);   // the previous sequence's queries are free
        if (!mbar_wait(&q_full[nseq & 1], (nseq >> 1) & 1, &s_abort)) break;
        cur_seq = s;
        ++nseq;
      }
      if (!mbar_wait(&full_bar[slot], par, &s_abort) || !mbar_wait(&acc_empty[as], apar ^ 1u, &s_abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t kd = kdesc0 + static_cast<uint64_t>((static_cast<long>(slot) * a.stage_bytes) >> 4);
      const uint64_t qd = qdesc0 + static_cast<uint64_t>((((nseq - 1) & 1) * q_bytes) >> 4);
      for (int hl = 0; hl < a.hg; ++hl) {
        const uint32_t d = tmem + static_cast<uint32_t>((as * a.hg + hl) * 16);
        const uint64_t kh = kd + static_cast<uint64_t>(hl * 1024);                  // 16 KiB per head tile
        const uint64_t qh = qd + static_cast<uint64_t>((g * a.hg + hl) * (IDXT_QHEAD >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16_ss(d, kh + kk * 2, qh + kk * 2, idesc, kk > 0 ? 1u : 0u);
      }
      umma_commit(&empty_bar[slot]);
      umma_commit(&acc_full[as]);
    }
    if (s_abort) {
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else if (nstage > 0 && warp >= 2) {
    // ------------------------------------------------------------ pooling warps: thread = key row
    // group G takes the stages k with k % IDXT_GROUPS == G; its 4 warps cover the 4 TMEM lane quarters
    const int G = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int token = q4 * 32 + lane;
    const int ptid = ((warp - 2) & 3) * 32 + lane;       // 0..127 within the group
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    int s, b;
    locate(u0, s, b);
    int cur_seq = -1, nq = 0, qrow0 = 0, ctx = 0;
    int pv_nq = 0, pv_row0 = 0, pv_g = 0, pv_b = 0;
    auto combine = [&](int pbuf) {                       // the group's previous stage: block scores
      if (ptid < pv_nq) {
        float tot = 0.f;
        for (int hl = 0; hl < a.hg; ++hl) {
          const uint32_t* pp = s_part[pbuf][ptid][hl];
          tot += key_to_float(max(max(pp[0], pp[1]), max(pp[2], pp[3])));
        }
        a.scores[(static_cast<long>(pv_row0 + ptid) * a.Hkv + pv_g) * a.max_blocks + pv_b] = tot;
      }
    };
    bool ok = true;
    int g = 0, as = 0, done = 0;
    uint32_t apar = 0;
    for (long k = 0; k < nstage; ++k) {
      if (k > 0) {
        if (++g == a.Hkv) { g = 0; advance(s, b); }
        if (++as == nslot) { as = 0; apar ^= 1u; }
      }
      if ((k % IDXT_GROUPS) != G) continue;
      if (s != cur_seq) {
        cur_seq = s;
        qrow0 = __ldg(a.q_start + s);
        nq = __ldg(a.q_start + s + 1) - qrow0;
        ctx = __ldg(a.ctx_len + s);
        if (nq > NQ) { if (ptid == 0) flag_error(MSA_DEV_BOUNDS); nq = NQ; }
      }
      // the group wait is also the barrier after which the group's previous partial maxima are visible
      if (!mbar_wait_group(&acc_full[as], apar, &s_abort, 1 + G, 128)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // every head's scores of this stage in flight at once, one wait
      float v[IDXT_MAXHG][16];
#pragma unroll
      for (int hl = 0; hl < IDXT_MAXHG; ++hl)
        if (hl < a.hg) tmem_ld16(lane_addr + static_cast<uint32_t>((as * a.hg + hl) * 16), v[hl]);
      if (done > 0) combine(((done - 1) & 1) * IDXT_GROUPS + G);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[as]);
      const int pbuf = (done & 1) * IDXT_GROUPS + G;      // alternates over the group's own stages
      const int j = b * a.block_size + token;            // absolute key position
#pragma unroll
      for (int hl = 0; hl < IDXT_MAXHG; ++hl) {
        if (hl < a.hg) {
#pragma unroll
          for (int i = 0; i < NQ; ++i) {
            if (i < nq) {
              const int p = ctx - nq + i;
              const uint32_t mx = __reduce_max_sync(0xFFFFFFFFu, order_key(j <= p ? v[hl][i] : -INFINITY));
              if (lane == 0) s_part[pbuf][i][hl][q4] = mx;
            }
          }
        }
      }
      pv_nq = nq; pv_row0 = qrow0; pv_g = g; pv_b = b;
      ++done;
    }
    if (ok && done > 0) {
      named_bar_sync(1 + G, 128);                        // the group's last partial maxima visible
      combine(((done - 1) & 1) * IDXT_GROUPS + G);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace msa
