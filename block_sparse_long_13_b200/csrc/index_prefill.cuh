// msa_index_scores, tensor-core form (prefill: many queries per sequence).
//
// Same definition as the streaming form:
//   S_g(r, b) = sum_{h in heads(g)} max_{j in block b, j <= p_r} q_h(r) . k_h(j)
// (inteligile "MiniMax-M3" model page, row "Indexer-selected sparse
// attention"; 24-ai.news, block scoring per query group).
//
// Work unit = (sequence, tile of 128 query rows, KV group g).  For each
// causally visible key block b the unit computes, per indexer head of the
// group, the 128 x 128 score tile Q_h K_h^T (K = 64) with tcgen05.mma into a
// TMEM accumulator, and four epilogue warps (thread = query row = TMEM lane)
// max-pool the row over the block's visible keys and sum over the heads.
//
// Roles: warp 0 = TMA producer (query tile once per unit, key tiles through a
// STAGES-deep ring), warp 1 = TMEM owner + single-thread UMMA issuer, warps
// 2..5 = epilogue.  Accumulators are double-buffered in TMEM (4 / hg
// buffers of hg x 128 fp32 columns) so the tensor core computes block b+1
// while the epilogue pools block b.  Units are dealt to persistent CTAs in
// snake order over a longest-first list (a query tile's cost grows with its
// position).
#pragma once
#include "common.cuh"

namespace msa {

constexpr int IDXP_THREADS = 192;
constexpr int IDXP_TILE = 128;
constexpr int IDXP_MAXSEQ = 1024;

struct IdxPrefillArgs {
  float* scores;             // [total_q][Hkv][max_blocks]
  const int32_t* q_start;
  const int32_t* ctx_len;
  const int32_t* page_table;
  int num_seqs, total_q, max_blocks, num_pages, Hi, Hkv, hg, block_size;
  int stages, nbuf;          // K ring depth; TMEM accumulator buffers
};

struct IdxUnit {
  int seq, row0, nrows, g, nblk;  // rows [row0, row0 + nrows); blocks 0 .. nblk-1
  int qs, nq, ctx;
};

__global__ void __launch_bounds__(IDXP_THREADS, 1)
index_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,   // idx_q  (64, Hi, total_q)
                     const __grid_constant__ CUtensorMap tmap_k,   // idx_k  (64, 128, Hi, P)
                     const IdxPrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const int head_bytes = IDXP_TILE * 64 * 2;            // 16 KiB per head tile
  const int q_bytes = a.hg * head_bytes;
  const int k_bytes = a.hg * head_bytes;
  uint8_t* q_smem = smem;
  uint8_t* k_smem = smem + q_bytes;

  __shared__ uint64_t k_full[8], k_empty[8], acc_full[4], acc_empty[4], q_full, q_empty, drain_bar;
  __shared__ uint32_t s_tmem;
  __shared__ int s_tprefix[IDXP_MAXSEQ + 1];
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    s_abort = 0;
    int acc = 0;
    s_tprefix[0] = 0;
    for (int s = 0; s < a.num_seqs; ++s) {
      const int nq = __ldg(a.q_start + s + 1) - __ldg(a.q_start + s);
      acc += (max(nq, 0) + IDXP_TILE - 1) / IDXP_TILE;
      s_tprefix[s + 1] = acc;
    }
    for (int i = 0; i < a.stages; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < a.nbuf; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    mbar_init(&drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {  // TMEM: 512 columns (the CTA is alone on its SM: > half the shared memory)
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  const int total_tiles = s_tprefix[a.num_seqs];
  const int total_units = total_tiles * a.Hkv;
  const int G = gridDim.x;

  // k-th unit of this CTA (snake order over the longest-first list); false when done
  auto get_unit = [&](int k, IdxUnit& u) -> bool {
    const int r = k;  // round
    const int c = blockIdx.x;
    const long idx = static_cast<long>(r) * G + ((r & 1) ? (G - 1 - c) : c);
    if (idx >= total_units) return false;
    const int tau = total_tiles - 1 - static_cast<int>(idx / a.Hkv);  // last tiles first
    u.g = static_cast<int>(idx % a.Hkv);
    int lo = 0, hi = a.num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tprefix[mid] <= tau) lo = mid; else hi = mid - 1;
    }
    u.seq = lo;
    u.qs = __ldg(a.q_start + lo);
    u.nq = __ldg(a.q_start + lo + 1) - u.qs;
    u.ctx = __ldg(a.ctx_len + lo);
    const int tin = tau - s_tprefix[lo];
    u.row0 = u.qs + tin * IDXP_TILE;
    u.nrows = min(IDXP_TILE, u.nq - tin * IDXP_TILE);
    const int p_last = u.ctx - u.nq + (u.row0 - u.qs) + u.nrows - 1;
    u.nblk = max(0, min(p_last / a.block_size + 1, a.max_blocks));
    if (p_last < 0) u.nblk = 0;
    return true;
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    uint32_t kit = 0, uit = 0;
    int last_parity[8];
    for (int i = 0; i < 8; ++i) last_parity[i] = -1;
    int q_parity = -1;
    IdxUnit u;
    for (int k = 0; get_unit(k, u) && !s_abort; ++k) {
      if (u.nblk == 0) continue;
      if (!mbar_wait(&q_empty, (uit & 1) ^ 1, &s_abort)) break;
      mbar_arrive_expect_tx(&q_full, q_bytes);
      for (int hl = 0; hl < a.hg; ++hl)
        tma_load_3d(q_smem + hl * head_bytes, &tmap_q, &q_full, 0, u.g * a.hg + hl, u.row0);
      q_parity = uit & 1;
      ++uit;
      bool ok = true;
      for (int b = 0; b < u.nblk; ++b, ++kit) {
        const int st = kit % a.stages;
        if (!mbar_wait(&k_empty[st], ((kit / a.stages) & 1) ^ 1, &s_abort)) { ok = false; break; }
        int page = __ldg(a.page_table + static_cast<long>(u.seq) * a.max_blocks + b);
        if (page < 0 || page >= a.num_pages) { flag_error(MSA_DEV_BOUNDS); page = 0; }
        mbar_arrive_expect_tx(&k_full[st], k_bytes);
        tma_load_4d(k_smem + st * k_bytes, &tmap_k, &k_full[st], 0, 0, u.g * a.hg, page);
        last_parity[st] = (kit / a.stages) & 1;
      }
      if (!ok) break;
    }
    if (s_abort) {  // let issued copies land before the CTA exits
      for (int i = 0; i < a.stages; ++i)
        if (last_parity[i] >= 0) mbar_wait_drain(&k_full[i], last_parity[i]);
      if (q_parity >= 0) mbar_wait_drain(&q_full, q_parity);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ UMMA issuer
    const uint32_t idesc = idesc_bf16(128, 128, false, false);
    const uint32_t q_addr = smem_u32(q_smem), k_addr = smem_u32(k_smem);
    uint32_t kit = 0, uit = 0, ait = 0;
    IdxUnit u;
    for (int k = 0; get_unit(k, u) && !s_abort; ++k) {
      if (u.nblk == 0) continue;
      if (!mbar_wait(&q_full, uit & 1, &s_abort)) break;
      ++uit;
      bool ok = true;
      for (int b = 0; b < u.nblk; ++b, ++kit, ++ait) {
        const int st = kit % a.stages;
        const int buf = ait % a.nbuf;
        if (!mbar_wait(&acc_empty[buf], ((ait / a.nbuf) & 1) ^ 1, &s_abort)) { ok = false; break; }
        if (!mbar_wait(&k_full[st], (kit / a.stages) & 1, &s_abort)) { ok = false; break; }
        tc_fence_after();
        for (int hl = 0; hl < a.hg; ++hl) {
          const uint32_t d = tmem + static_cast<uint32_t>((buf * a.hg + hl) * 128);
          const uint32_t qa = q_addr + hl * head_bytes;
          const uint32_t ka = k_addr + st * k_bytes + hl * head_bytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ss(d, sdesc_sw128(qa + kk * 32, 16, 1024), sdesc_sw128(ka + kk * 32, 16, 1024), idesc,
                         kk > 0 ? 1u : 0u);
        }
        umma_commit(&k_empty[st]);
        umma_commit(&acc_full[buf]);
      }
      umma_commit(&q_empty);  // the query tile is free once this unit's MMAs are done
      if (!ok) break;
    }
    if (s_abort) {
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;         // row of the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t ait = 0;
    IdxUnit u;
    for (int k = 0; get_unit(k, u); ++k) {  // exits are warp-uniform
      if (u.nblk == 0) continue;
      const bool valid = r < u.nrows;
      const int row = u.row0 + r;
      const int p = u.ctx - u.nq + (row - u.qs);
      float* srow = a.scores + (static_cast<long>(row) * a.Hkv + u.g) * a.max_blocks;
      bool ok = true;
      for (int b = 0; b < u.nblk; ++b, ++ait) {
        const int buf = ait % a.nbuf;
        if (!mbar_wait_warp(&acc_full[buf], (ait / a.nbuf) & 1, &s_abort)) { ok = false; break; }
        tc_fence_after();
        const int vis = p - b * a.block_size + 1;   // visible keys of block b for this row
        float tot = 0.f;
        for (int hl = 0; hl < a.hg; ++hl) {
          float mx = -INFINITY;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float v0[32], v1[32];
            const uint32_t col = static_cast<uint32_t>((buf * a.hg + hl) * 128 + half * 64);
            tmem_ld32(lane_addr + col, v0);
            tmem_ld32(lane_addr + col + 32, v1);
            tmem_ld_wait();
            const int base = half * 64;
            if (vis >= base + 64) {
#pragma unroll
              for (int c = 0; c < 32; ++c) mx = fmaxf(mx, fmaxf(v0[c], v1[c]));
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                if (base + c < vis) mx = fmaxf(mx, v0[c]);
                if (base + 32 + c < vis) mx = fmaxf(mx, v1[c]);
              }
            }
          }
          tot += mx;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        if (valid) srow[b] = tot;  // -inf when the block is past the row's current block
      }
      if (!ok) break;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace msa
