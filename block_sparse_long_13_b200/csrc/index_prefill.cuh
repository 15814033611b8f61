// msa_index_scores, tensor-core form (prefill: many queries per sequence).
//
// Same definition as the streaming form:
//   S_g(r, b) = sum_{h in heads(g)} max_{j in block b, j <= p_r} q_h(r) . k_h(j)
// (inteligile "MiniMax-M3" model page, row "Indexer-selected sparse
// attention"; 24-ai.news, block scoring per query group).
//
// Work unit = (sequence, tile of 128 query rows, KV group g).  The unit walks
// its causally visible key blocks in pairs; one step = (block pair, indexer
// head h of the group): a single 128 x 256 x 64 product Q_h [K_h(b) ; K_h(b+1)]^T
// on tcgen05 into a 256-column TMEM accumulator (N = 256 keeps the 1-SM tensor
// core at full rate; N = 128 runs it at half rate).  Two epilogue warpgroups
// read every step, one block of the pair each (thread = query row = TMEM
// lane), max-pool the row over the block's visible keys and sum the group's
// heads in registers before writing the block score.
//
// Roles: warp 0 = TMA producer (query tiles double-buffered, key tiles of a
// (pair, head) through a ring), warp 1 = TMEM owner + single-thread UMMA
// issuer, warps 4..7 / 8..11 = the two epilogue warpgroups.  Accumulators are
// double-buffered (2 x 256 columns).  Units are dealt to persistent CTAs in a
// snake order over a longest-first list, group-major so that one group's keys
// are live in L2 at a time.
#pragma once
#include "common.cuh"

namespace msa {

constexpr int IDXP_THREADS = 384;   // warpgroup 0: producer + UMMA warps; warpgroups 1, 2: epilogue
// Register split (setmaxnreg; registers are granted per warpgroup): the launch gives 168 per thread
// (65536 / 384, rounded to 8); warpgroup 0 returns registers, the epilogue warpgroups take them.
constexpr int IDXP_REGS_CTRL = 72, IDXP_REGS_EPI = 216;
static_assert(128 * IDXP_REGS_CTRL + 256 * IDXP_REGS_EPI <= 384 * 168, "register split exceeds the launch");
constexpr int IDXP_TILE = 128;
constexpr int IDXP_MAXSEQ = 1024;
constexpr int IDXP_STAGE_BYTES = 2 * IDXP_TILE * 64 * 2;   // keys of one head for two blocks: 32 KiB

constexpr int IDXP_FUSED_SLOTS = 15;   // fused top-k: candidate slots per row (topk <= 16)

struct IdxPrefillArgs {
  float* scores;             // [total_q][Hkv][max_blocks] (score form)
  int32_t* block_idx;        // [total_q][Hkv][topk] (fused form)
  int topk;
  const int32_t* q_start;
  const int32_t* ctx_len;
  const int32_t* page_table;
  int num_seqs, total_q, max_blocks, num_pages, Hi, Hkv, hg, block_size;
  int stages, nqbuf;         // key ring depth; query tile buffers
  int nsplit;                // pieces per (query tile, group) along its key blocks (1 in the fused form)
};

struct IdxUnit {
  int seq, row0, nrows, g, nblk;  // rows [row0, row0 + nrows); the tile sees blocks 0 .. nblk-1
  int qs, nq, ctx;
  int pr0, npr;                   // this piece: block pairs pr0 .. pr0+npr-1
};

// FUSED = false: write every block score.  FUSED = true: keep, per row, the best topk-1 earlier blocks
// by (score desc, block asc) in registers while the blocks stream by (each epilogue warpgroup sees
// half of them), merge the two halves through shared memory at the end of the unit and write the
// selection (ascending, the row's own block included, -1 padded): the same rule and the same fp32
// scores as msa_topk_blocks, without materialising the score matrix.
template <bool FUSED>
__global__ void __launch_bounds__(IDXP_THREADS, 1)
index_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,   // idx_q  (64, Hi, total_q), box (64, 1, 128)
                     const __grid_constant__ CUtensorMap tmap_k,   // idx_k  (64, P*Hi*128), box (64, 128)
                     const IdxPrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const int head_bytes = IDXP_TILE * 64 * 2;            // 16 KiB per head tile
  const int q_bytes = a.hg * head_bytes;
  uint8_t* q_smem = smem;
  uint8_t* k_smem = smem + a.nqbuf * q_bytes;

  __shared__ uint64_t k_full[8], k_empty[8], acc_full[2], acc_empty[2], q_full[2], q_empty[2], drain_bar;
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 8);       // both epilogue warpgroups read every step
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
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
  const long total_units = static_cast<long>(total_tiles) * a.Hkv * a.nsplit;
  const int G = gridDim.x;

  // k-th unit of this CTA (snake order over the longest-first list); false when done.  A unit is one of
  // the nsplit pieces of a (query tile, group) along its key blocks: block scores need no reduction
  // across blocks, and causal tiles differ in length, so whole tiles over the persistent CTAs left the
  // last wave of units 20-60 % unbalanced.
  auto get_unit = [&](int k, IdxUnit& u) -> bool {
    const int c = blockIdx.x;
    const long idx = static_cast<long>(k) * G + ((k & 1) ? (G - 1 - c) : c);
    if (idx >= total_units) return false;
    const int piece = static_cast<int>(idx % a.nsplit);
    const long tidx = idx / a.nsplit;
    // group-major: all CTAs work on one group's keys at a time (they stay in L2);
    // within a group the last (longest) query tiles come first
    u.g = static_cast<int>(tidx / total_tiles);
    const int tau = total_tiles - 1 - static_cast<int>(tidx % total_tiles);
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
    const int npair = (u.nblk + 1) >> 1;
    u.pr0 = static_cast<int>(static_cast<long>(piece) * npair / a.nsplit);
    u.npr = static_cast<int>(static_cast<long>(piece + 1) * npair / a.nsplit) - u.pr0;
    return true;
  };

  if (warp < 4) {
  regs_dec<IDXP_REGS_CTRL>();   // warps 2 and 3 have no role; they wait at the final barrier
  if (warp == 0) {
    // ------------------------------------------------------------ producer warp
    // lane 0 issues the copies; the whole warp reads the page ids of the next 32 blocks at once
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
    }
    uint32_t kit = 0, uit = 0;
    uint32_t used = 0, parity_bits = 0;   // key ring slots: issued at least once / parity of the last issue
    const uint64_t pol_k = l2_policy_evict_last();   // a group's keys are read by every query tile
    int q_parity0 = -1, q_parity1 = -1;
    IdxUnit u;
    for (int k = 0; get_unit(k, u) && !s_abort; ++k) {
      if (u.npr == 0) continue;
      const int qb = uit % a.nqbuf;
      const uint32_t qpar = (uit / a.nqbuf) & 1;
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&q_empty[qb], qpar ^ 1, &s_abort);
        if (ok) {
          mbar_arrive_expect_tx(&q_full[qb], q_bytes);
          for (int hl = 0; hl < a.hg; ++hl)
            tma_load_3d(q_smem + qb * q_bytes + hl * head_bytes, &tmap_q, &q_full[qb], 0, u.g * a.hg + hl, u.row0);
          if (qb == 0) q_parity0 = static_cast<int>(qpar); else q_parity1 = static_cast<int>(qpar);
        }
      }
      if (__any_sync(0xFFFFFFFFu, !ok)) break;
      ++uit;
      int page_l = 0;
      for (int pr = u.pr0; pr < u.pr0 + u.npr && ok; ++pr) {
        const int b0 = 2 * pr;
        if ((b0 & 31) == 0 || pr == u.pr0) {  // page ids of the 32-block window holding b0 and b0+1
          const int bb = (b0 & ~31) + lane;
          page_l = 0;
          if (bb < u.nblk) {
            page_l = __ldg(a.page_table + static_cast<long>(u.seq) * a.max_blocks + bb);
            if (page_l < 0 || page_l >= a.num_pages) { flag_error(MSA_DEV_BOUNDS); page_l = 0; }
          }
        }
        const int page0 = __shfl_sync(0xFFFFFFFFu, page_l, b0 & 31);
        int page1 = __shfl_sync(0xFFFFFFFFu, page_l, (b0 + 1) & 31);
        if (b0 + 1 >= u.nblk) page1 = page0;  // odd block count: the second half is ignored
        for (int hl = 0; hl < a.hg; ++hl, ++kit) {
          const int st = kit % a.stages;
          if (lane == 0) {
            ok = mbar_wait(&k_empty[st], ((kit / a.stages) & 1) ^ 1, &s_abort);
            if (ok) {
              uint8_t* dst = k_smem + st * IDXP_STAGE_BYTES;
              mbar_arrive_expect_tx(&k_full[st], IDXP_STAGE_BYTES);
              const int h = u.g * a.hg + hl;    // key rows of (page, head): one contiguous 16 KiB box
              tma_load_2d_hint(dst, &tmap_k, &k_full[st], 0, (page0 * a.Hi + h) * 128, pol_k);
              tma_load_2d_hint(dst + head_bytes, &tmap_k, &k_full[st], 0, (page1 * a.Hi + h) * 128, pol_k);
              used |= 1u << st;
              parity_bits = (parity_bits & ~(1u << st)) | (((kit / a.stages) & 1u) << st);
            }
          }
          if (__any_sync(0xFFFFFFFFu, !ok)) { ok = false; break; }
        }
      }
      if (!ok) break;
    }
    if (lane == 0 && s_abort) {  // let issued copies land before the CTA exits
      for (int i = 0; i < a.stages; ++i)
        if (used & (1u << i)) mbar_wait_drain(&k_full[i], (parity_bits >> i) & 1u);
      if (q_parity0 >= 0) mbar_wait_drain(&q_full[0], q_parity0);
      if (q_parity1 >= 0) mbar_wait_drain(&q_full[1], q_parity1);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ UMMA issuer
    // One thread issues everything, so its own instruction latency is on the critical path: the
    // descriptors are built once (only the 14-bit start address, in 16-byte units, moves between
    // MMAs) and the ring positions are counters, not divisions.
    const uint32_t idesc = idesc_bf16(128, 256, false, false);
    const uint64_t qdesc0 = sdesc_sw128(smem_u32(q_smem), 16, 1024);
    const uint64_t kdesc0 = sdesc_sw128(smem_u32(k_smem), 16, 1024);
    int st = 0, buf = 0;                    // key stage, accumulator buffer
    uint32_t kph = 0, aph = 0;              // phase of the key ring's current lap; accumulator use count / 2
    uint32_t uit = 0;
    IdxUnit u;
    for (int k = 0; get_unit(k, u) && !s_abort; ++k) {
      if (u.npr == 0) continue;
      const int qb = a.nqbuf == 1 ? 0 : static_cast<int>(uit & 1);
      const uint32_t qpar = a.nqbuf == 1 ? (uit & 1) : ((uit >> 1) & 1);
      if (!mbar_wait(&q_full[qb], qpar, &s_abort)) break;
      ++uit;
      // The tensor pipe queues about one MMA: the barriers of step sp + 1 are awaited while the first
      // two MMAs of step sp run, so the next step's MMAs are ready when the pipe frees up.
      const int nstep = u.npr * a.hg;
      bool ok = nstep > 0 && mbar_wait(&acc_empty[buf], (aph & 1) ^ 1, &s_abort) && mbar_wait(&k_full[st], kph, &s_abort);
      int hl = 0;
      for (int sp = 0; sp < nstep && ok; ++sp) {
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf * 256);
        const uint64_t qd = qdesc0 + static_cast<uint64_t>((qb * q_bytes + hl * head_bytes) >> 4);
        const uint64_t kd = kdesc0 + static_cast<uint64_t>((st * IDXP_STAGE_BYTES) >> 4);   // two blocks
        umma_bf16_ss(d, qd, kd, idesc, 0u);
        umma_bf16_ss(d, qd + 2, kd + 2, idesc, 1u);
        // positions of the next step, and its barriers
        int st2 = st + 1;
        uint32_t kph2 = kph;
        if (st2 == a.stages) { st2 = 0; kph2 ^= 1u; }
        const int buf2 = buf ^ 1;
        const uint32_t aph2 = aph + static_cast<uint32_t>(buf);
        if (sp + 1 < nstep)
          ok = mbar_wait(&acc_empty[buf2], (aph2 & 1) ^ 1, &s_abort) && mbar_wait(&k_full[st2], kph2, &s_abort);
        umma_bf16_ss(d, qd + 4, kd + 4, idesc, 1u);
        umma_bf16_ss(d, qd + 6, kd + 6, idesc, 1u);
        umma_commit(&k_empty[st]);
        umma_commit(&acc_full[buf]);
        st = st2;
        kph = kph2;
        buf = buf2;
        aph = aph2;
        if (++hl == a.hg) hl = 0;
      }
      umma_commit(&q_empty[qb]);  // the query tile is free once this unit's MMAs are done
      if (!ok) break;
    }
    if (s_abort) {
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  }
  } else {
    regs_inc<IDXP_REGS_EPI>();
    // ------------------------------------------------------------ epilogue warpgroups
    const int w = (warp - 4) >> 2;             // this warpgroup pools block 2*pair + w of every step
    const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;         // row of the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t ait = 0;
    IdxUnit u;
    for (int k = 0; get_unit(k, u); ++k) {     // exits are warp-uniform
      if (u.npr == 0) continue;
      const bool valid = r < u.nrows;
      const int row = u.row0 + r;
      const int p = u.ctx - u.nq + (row - u.qs);
      float* srow = FUSED ? nullptr : a.scores + (static_cast<long>(row) * a.Hkv + u.g) * a.max_blocks;
      const int nstep = u.npr * a.hg;
      bool ok = true;
      float tot = 0.f;
      // fused form: candidate keys (order_key(score) << 32 | ~block); unused slots hold ~0 and are never
      // replaced, so kmin is the smallest key among the topk-1 live slots (0 = empty)
      const int cur_blk = p >= 0 ? p / a.block_size : -1;
      uint64_t ck[IDXP_FUSED_SLOTS];
      uint64_t kmin = 0;
      int kpos = 0;
      if (FUSED) {
#pragma unroll
        for (int i = 0; i < IDXP_FUSED_SLOTS; ++i) ck[i] = i < a.topk - 1 ? 0ull : ~0ull;
        kmin = a.topk > 1 ? 0ull : ~0ull;
      }
      auto insert = [&](uint64_t key) {          // replace the smallest live slot with key (key > kmin)
#pragma unroll
        for (int i = 0; i < IDXP_FUSED_SLOTS; ++i)
          if (i == kpos) ck[i] = key;
        kmin = ck[0];
        kpos = 0;
#pragma unroll
        for (int i = 1; i < IDXP_FUSED_SLOTS; ++i)
          if (ck[i] < kmin) { kmin = ck[i]; kpos = i; }
      };
      // head hl of the group and this warpgroup's block b of step sp, kept as counters: a runtime
      // division per step sits on this loop's dependency chain
      int hl = 0, b = 2 * u.pr0 + w;
      for (int sp = 0; sp < nstep; ++sp, ++ait) {
        if (sp > 0 && ++hl == a.hg) { hl = 0; b += 2; }
        const int buf = ait & 1;
        if (!mbar_wait_warp(&acc_full[buf], (ait >> 1) & 1, &s_abort)) { ok = false; break; }
        tc_fence_after();
        float v0[32], v1[32], v2[32], v3[32];  // the block's 128 scores for this row
        const uint32_t col = lane_addr + static_cast<uint32_t>(buf * 256 + w * 128);
        tmem_ld32(col, v0);
        tmem_ld32(col + 32, v1);
        tmem_ld32(col + 64, v2);
        tmem_ld32(col + 96, v3);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        const int vis = p - b * a.block_size + 1;   // visible keys of block b for this row
        float mx[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
        if (vis >= 128) {
#pragma unroll
          for (int c = 0; c < 32; ++c) mx[c & 7] = fmax3(fmax3(mx[c & 7], v0[c], v1[c]), v2[c], v3[c]);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c < vis) mx[c & 7] = fmaxf(mx[c & 7], v0[c]);
            if (32 + c < vis) mx[c & 7] = fmaxf(mx[c & 7], v1[c]);
            if (64 + c < vis) mx[c & 7] = fmaxf(mx[c & 7], v2[c]);
            if (96 + c < vis) mx[c & 7] = fmaxf(mx[c & 7], v3[c]);
          }
        }
        const float hm = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], fmax3(mx[4], mx[5], mx[6]), mx[7]));
        tot = (hl == 0) ? hm : tot + hm;
        if (FUSED) {
          if (hl == a.hg - 1 && valid && b < cur_blk && tot > -INFINITY) {   // candidates: earlier blocks
            const uint64_t key = (static_cast<uint64_t>(order_key(tot)) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(b));
            if (key > kmin) insert(key);
          }
        } else if (hl == a.hg - 1 && valid && b < u.nblk) {
          __stcs(srow + b, tot);                 // -inf past the row's block
        }
      }
      if (FUSED) {
        // merge the two warpgroups' halves: warp (4 + quarter) and warp (8 + quarter) own the same rows
        uint64_t* xb = reinterpret_cast<uint64_t*>(k_smem + a.stages * IDXP_STAGE_BYTES) + r * IDXP_FUSED_SLOTS;
        if (w == 1) {
#pragma unroll
          for (int i = 0; i < IDXP_FUSED_SLOTS; ++i) xb[i] = ck[i];
        }
        if (named_bar_any(1 + quarter, 64, !ok)) break;   // both warps of the pair leave together
        if (w == 0) {
#pragma unroll
          for (int i = 0; i < IDXP_FUSED_SLOTS; ++i) {
            const uint64_t key = xb[i];
            if (key != ~0ull && key > kmin) insert(key);
          }
        }
        named_bar_sync(1 + quarter, 64);        // the partner may refill the buffer for its next unit
        if (w == 0 && valid) {
          int32_t* orow = a.block_idx + (static_cast<long>(row) * a.Hkv + u.g) * a.topk;
          if (cur_blk < 0 || cur_blk >= a.max_blocks) {
            flag_error(MSA_DEV_BOUNDS);
            for (int j = 0; j < a.topk; ++j) orow[j] = -1;
          } else {
            int nsel = 0;
#pragma unroll
            for (int i = 0; i < IDXP_FUSED_SLOTS; ++i) nsel += (ck[i] != 0ull && ck[i] != ~0ull) ? 1 : 0;
#pragma unroll
            for (int i = 0; i < IDXP_FUSED_SLOTS; ++i) {
              if (ck[i] != 0ull && ck[i] != ~0ull) {
                const uint32_t bi = 0xFFFFFFFFu - static_cast<uint32_t>(ck[i]);
                int rank = 0;                    // ids are distinct: rank = number of smaller ids
#pragma unroll
                for (int j = 0; j < IDXP_FUSED_SLOTS; ++j)
                  rank += (ck[j] != 0ull && ck[j] != ~0ull && 0xFFFFFFFFu - static_cast<uint32_t>(ck[j]) < bi) ? 1 : 0;
                orow[rank] = static_cast<int32_t>(bi);
              }
            }
            orow[nsel] = cur_blk;                // every candidate lies before the row's own block
            for (int j = nsel + 1; j < a.topk; ++j) orow[j] = -1;
          }
        }
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
