// msa_attn_prefill: block-major ("KV outer, gather Q") sparse GQA attention.
//
// shaam.blog, "What makes MiniMax M3 different ...": each KV block is read
// once with contiguous access and the queries that chose it are gathered;
// daily.dev "Serving options": KV-block-major prefill scheduling; inteligile
// tags "Two-phase forward", "LSE fusion", "query concatenation".
//
// Phase 0 (schedule): invert the selections.  Every (row t, group g, slot)
// with block_idx[t][g][slot] = b >= 0 is an entry of bucket (seq, g, b);
// count -> exclusive scan -> scatter gives each bucket its entry list, cut
// into tiles of at most 8 entries.
//
// Phase 1 (this file's tensor-core kernel): a tile stacks the 16 query heads
// of its <= 8 gathered tokens into the 128 rows of one MMA ("query
// concatenation").  K_b and V_b (128 x 128 bf16 each, one TMA load per
// bucket per CTA) stay in shared memory while the CTA walks consecutive
// tiles of the same bucket.  S = Q K^T and O = P V run on tcgen05 with fp32
// accumulators in TMEM; a 4-warp softmax group reads S rows from TMEM (thread
// = row), masks keys after the query position (only the query's own block
// has any), writes P as bf16 into a swizzled shared tile, and later stores
// O / l (bf16) and lse = m + ln l as the partial of (t, head, slot).
//
// Phase 2 (merge): out(t, h) = sum_slots exp(lse_s - L) O_s with
// L = log sum_s exp(lse_s); lse(t, h) = L.
#pragma once
#include "common.cuh"

namespace msa {

constexpr int ATTP_THREADS = 192;
constexpr int ATTP_TOK = 8;       // tokens per tile (x 16 heads = 128 MMA rows)
constexpr int ATTP_G = 16;        // query heads per KV group
constexpr int SCHED_ROWS = 256;   // query rows per schedule CTA
constexpr int SCHED_SMEM_BUCKETS = 4096;

// ------------------------------------------------------------------ schedule
struct SchedArgs {
  const int32_t* block_idx;   // [total_q][Hkv][topk]
  const int32_t* q_start;
  const int32_t* ctx_len;
  int* counts;                // [nbuckets]          (zeroed by the host before count)
  int* offsets;               // [nbuckets + 1]
  int* tile_offsets;          // [nbuckets + 1]
  int* cursor;                // [nbuckets]
  int* entries;               // [total_q * Hkv * topk]  (t << 6) | slot
  int* total_tiles;           // [1]
  int num_seqs, total_q, Hkv, topk, max_blocks, block_size, nbuckets;
};

__device__ __forceinline__ int entry_bucket(const SchedArgs& a, int t, int g, int b, int s) {
  return (s * a.Hkv + g) * a.max_blocks + b;
}

// pass = 0: count entries per bucket; pass = 1: scatter them
__global__ void __launch_bounds__(256) sched_count_scatter_kernel(const SchedArgs a, int pass) {
  extern __shared__ int sh[];  // [3][nbuckets] when nbuckets <= SCHED_SMEM_BUCKETS
  const bool use_smem = a.nbuckets <= SCHED_SMEM_BUCKETS;
  int* lcnt = sh;
  int* lbase = sh + a.nbuckets;
  int* lcur = sh + 2 * a.nbuckets;
  const int t0 = blockIdx.x * SCHED_ROWS;
  const int t1 = min(a.total_q, t0 + SCHED_ROWS);
  if (use_smem) {
    for (int i = threadIdx.x; i < a.nbuckets; i += blockDim.x) { lcnt[i] = 0; lcur[i] = 0; }
    __syncthreads();
  }
  const int per_row = a.Hkv * a.topk;
  const long e0 = static_cast<long>(t0) * per_row, e1 = static_cast<long>(t1) * per_row;
  // entries of this CTA's rows
  for (int round = 0; round < (use_smem && pass == 1 ? 2 : 1); ++round) {
    for (long e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
      const int b = __ldg(a.block_idx + e);
      if (b < 0) continue;
      const int t = static_cast<int>(e / per_row);
      const int g = static_cast<int>((e / a.topk) % a.Hkv);
      const int slot = static_cast<int>(e % a.topk);
      const int s = find_seq(a.q_start, a.num_seqs, t);
      const int qs = __ldg(a.q_start + s), nq = __ldg(a.q_start + s + 1) - qs;
      const int p = __ldg(a.ctx_len + s) - nq + (t - qs);
      if (b >= a.max_blocks || b > p / a.block_size) { flag_error(MSA_DEV_BOUNDS); continue; }
      const int bk = entry_bucket(a, t, g, b, s);
      if (pass == 0) {
        if (use_smem) atomicAdd(&lcnt[bk], 1); else atomicAdd(&a.counts[bk], 1);
      } else if (!use_smem) {
        const int pos = atomicAdd(&a.cursor[bk], 1);
        a.entries[pos] = (t << 6) | slot;
      } else if (round == 0) {
        atomicAdd(&lcnt[bk], 1);
      } else {
        const int pos = lbase[bk] + atomicAdd(&lcur[bk], 1);
        a.entries[pos] = (t << 6) | slot;
      }
    }
    if (use_smem) {
      __syncthreads();
      if (pass == 0) {
        for (int i = threadIdx.x; i < a.nbuckets; i += blockDim.x)
          if (lcnt[i]) atomicAdd(&a.counts[i], lcnt[i]);
      } else if (round == 0) {
        for (int i = threadIdx.x; i < a.nbuckets; i += blockDim.x)
          if (lcnt[i]) lbase[i] = atomicAdd(&a.cursor[i], lcnt[i]);
        __syncthreads();
      }
    }
  }
}

// one CTA: exclusive scans of entry counts and of tiles per bucket, packed as
// (tiles << 32 | entries) in 64-bit sums (entries per call < 2^31)
__global__ void __launch_bounds__(1024) sched_scan_kernel(const SchedArgs a) {
  __shared__ unsigned long long s_w[32];
  __shared__ unsigned long long s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < a.nbuckets; base += 1024) {
    const int i = base + tid;
    const int c = i < a.nbuckets ? a.counts[i] : 0;
    const int tl = (c + ATTP_TOK - 1) / ATTP_TOK;
    const unsigned long long mine = (static_cast<unsigned long long>(tl) << 32) | static_cast<unsigned>(c);
    unsigned long long v = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long n = __shfl_up_sync(0xFFFFFFFFu, v, o);
      if (lane >= o) v += n;
    }
    if (lane == 31) s_w[warp] = v;
    __syncthreads();
    if (warp == 0) {
      unsigned long long w = s_w[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long n = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) w += n;
      }
      s_w[lane] = w;
    }
    __syncthreads();
    const unsigned long long ex = s_carry + (warp > 0 ? s_w[warp - 1] : 0ull) + v - mine;
    if (i < a.nbuckets) {
      a.offsets[i] = static_cast<int>(ex & 0xFFFFFFFFull);
      a.cursor[i] = static_cast<int>(ex & 0xFFFFFFFFull);
      a.tile_offsets[i] = static_cast<int>(ex >> 32);
    }
    __syncthreads();
    if (tid == 0) s_carry += s_w[31];
    __syncthreads();
  }
  if (tid == 0) {
    a.offsets[a.nbuckets] = static_cast<int>(s_carry & 0xFFFFFFFFull);
    a.tile_offsets[a.nbuckets] = static_cast<int>(s_carry >> 32);
    a.total_tiles[0] = static_cast<int>(s_carry >> 32);
  }
}

// ------------------------------------------------------------------ phase 1
struct AttnPrefillArgs {
  const int32_t* q_start;
  const int32_t* ctx_len;
  const int32_t* page_table;
  const int* offsets;        // [nbuckets + 1]
  const int* tile_offsets;   // [nbuckets + 1]
  const int* entries;
  const int* total_tiles;
  float* part_lse;           // [total_q][Hq][topk]
  int num_seqs, total_q, Hq, Hkv, topk, max_blocks, num_pages, block_size, nbuckets;
  float scale_log2;
};

struct TileInfo {
  int bucket, seq, g, b, e0, n;  // entries [e0, e0 + n)
};

__device__ __forceinline__ void tile_info(const AttnPrefillArgs& a, int tile, TileInfo& ti) {
  int lo = 0, hi = a.nbuckets - 1;  // largest bucket with tile_offsets[bucket] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(a.tile_offsets + mid) <= tile) lo = mid; else hi = mid - 1;
  }
  ti.bucket = lo;
  ti.b = lo % a.max_blocks;
  ti.g = (lo / a.max_blocks) % a.Hkv;
  ti.seq = lo / (a.max_blocks * a.Hkv);
  const int within = tile - __ldg(a.tile_offsets + lo);
  const int beg = __ldg(a.offsets + lo), end = __ldg(a.offsets + lo + 1);
  ti.e0 = beg + within * ATTP_TOK;
  ti.n = min(ATTP_TOK, end - ti.e0);
}

// shared memory plan (bytes, 1024-aligned): Q[2] 64K | K 32K | V 32K | P[2] 64K | O staging 32K
constexpr int ATTP_QBYTES = 32768, ATTP_KVBYTES = 32768;
constexpr int ATTP_SMEM = 2 * ATTP_QBYTES + 2 * ATTP_KVBYTES + 2 * 32768 + 32768 + 1024;

__global__ void __launch_bounds__(ATTP_THREADS, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,     // q as [total_q*Hq][128]
                    const __grid_constant__ CUtensorMap tmap_k,     // k as [P*Hkv*128][128]
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_po,    // partial O as [total_q*topk*Hq][128]
                    const AttnPrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;                                  // 2 x 32 KiB: [half][128 rows][64]
  uint8_t* k_s = q_s + 2 * ATTP_QBYTES;                 // [half][128 keys][64]
  uint8_t* v_s = k_s + ATTP_KVBYTES;                    // [half][128 keys][64]
  uint8_t* p_s = v_s + ATTP_KVBYTES;                    // 2 x 32 KiB: [half][128 rows][64 keys]
  uint8_t* o_s = p_s + 2 * 32768;                       // [half][128 rows][64]

  __shared__ uint64_t kv_full, kv_empty, q_full[2], q_empty[2], s_full[2], s_empty[2], p_full[2], p_empty[2],
      o_full[2], o_empty[2], drain_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_ent[3][ATTP_TOK];   // (t << 6 | slot) of each entry of the last three tiles

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    s_abort = 0;
    mbar_init(&kv_full, 1);
    mbar_init(&kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_empty[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 4);
    }
    mbar_init(&drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);  // S[2] at columns 0/128, O[2] at 256/384
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  const int T = __ldg(a.total_tiles);
  const int tile0 = static_cast<int>(static_cast<long>(T) * blockIdx.x / gridDim.x);
  const int tile1 = static_cast<int>(static_cast<long>(T) * (blockIdx.x + 1) / gridDim.x);
  const int ntile = tile1 - tile0;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    int cur_bucket = -1;
    uint32_t kvit = 0;
    int kv_parity = -1, qpar[2] = {-1, -1};
    for (int i = 0; i < ntile && !s_abort; ++i) {
      TileInfo ti;
      tile_info(a, tile0 + i, ti);
      if (ti.bucket != cur_bucket) {
        if (!mbar_wait(&kv_empty, (kvit & 1) ^ 1, &s_abort)) break;
        int page = __ldg(a.page_table + static_cast<long>(ti.seq) * a.max_blocks + ti.b);
        if (page < 0 || page >= a.num_pages) { flag_error(MSA_DEV_BOUNDS); page = 0; }
        const int y = (page * a.Hkv + ti.g) * 128;
        mbar_arrive_expect_tx(&kv_full, 2 * ATTP_KVBYTES);
        tma_load_2d(k_s, &tmap_k, &kv_full, 0, y);
        tma_load_2d(k_s + 16384, &tmap_k, &kv_full, 64, y);
        tma_load_2d(v_s, &tmap_v, &kv_full, 0, y);
        tma_load_2d(v_s + 16384, &tmap_v, &kv_full, 64, y);
        kv_parity = kvit & 1;
        ++kvit;
        cur_bucket = ti.bucket;
      }
      const int qb = i & 1;
      if (!mbar_wait(&q_empty[qb], ((i >> 1) & 1) ^ 1, &s_abort)) break;
      mbar_arrive_expect_tx(&q_full[qb], ti.n * 4096);
      for (int e = 0; e < ti.n; ++e) {
        const int ent = __ldg(a.entries + ti.e0 + e);
        const int t = ent >> 6;
        const int y = t * a.Hq + ti.g * ATTP_G;
        tma_load_2d(q_s + qb * ATTP_QBYTES + e * 2048, &tmap_q, &q_full[qb], 0, y);
        tma_load_2d(q_s + qb * ATTP_QBYTES + 16384 + e * 2048, &tmap_q, &q_full[qb], 64, y);
      }
      qpar[qb] = (i >> 1) & 1;
    }
    if (s_abort) {
      if (kv_parity >= 0) mbar_wait_drain(&kv_full, kv_parity);
      for (int j = 0; j < 2; ++j) if (qpar[j] >= 0) mbar_wait_drain(&q_full[j], qpar[j]);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ UMMA issuer
    const uint32_t id_s = idesc_bf16(128, 128, false, false);
    const uint32_t id_pv = idesc_bf16(128, 128, false, true);
    const uint32_t qa = smem_u32(q_s), ka = smem_u32(k_s), va = smem_u32(v_s), pa = smem_u32(p_s);
    int cur_bucket = -1;
    uint32_t kvit = 0;
    bool pv_pending = false;
    auto issue_pv = [&](int j) -> bool {  // O[j%2] = P[j%2] V
      const int pb = j & 1;
      if (!mbar_wait(&p_full[pb], (j >> 1) & 1, &s_abort)) return false;
      if (!mbar_wait(&o_empty[pb], ((j >> 1) & 1) ^ 1, &s_abort)) return false;
      tc_fence_after();
      const uint32_t d = tmem + 256 + pb * 128;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t adesc = sdesc_sw128(pa + pb * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t bdesc = sdesc_sw128(va + kk * 2048, 16384, 1024);
        umma_bf16_ss(d, adesc, bdesc, id_pv, kk > 0 ? 1u : 0u);
      }
      umma_commit(&o_full[pb]);
      umma_commit(&p_empty[pb]);
      return true;
    };
    bool ok = true;
    for (int i = 0; i < ntile && ok && !s_abort; ++i) {
      TileInfo ti;
      tile_info(a, tile0 + i, ti);
      if (ti.bucket != cur_bucket) {
        if (pv_pending) {  // finish the previous bucket before its K/V is replaced
          if (!issue_pv(i - 1)) break;
          pv_pending = false;
        }
        if (cur_bucket >= 0) umma_commit(&kv_empty);
        if (!mbar_wait(&kv_full, kvit & 1, &s_abort)) break;
        ++kvit;
        cur_bucket = ti.bucket;
      }
      const int qb = i & 1;
      if (!mbar_wait(&q_full[qb], (i >> 1) & 1, &s_abort)) break;
      if (!mbar_wait(&s_empty[qb], ((i >> 1) & 1) ^ 1, &s_abort)) break;
      tc_fence_after();
      const uint32_t d = tmem + qb * 128;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        umma_bf16_ss(d, sdesc_sw128(qa + qb * ATTP_QBYTES + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), id_s,
                     kk > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[qb]);
      umma_commit(&q_empty[qb]);
      if (pv_pending) ok = issue_pv(i - 1);
      pv_pending = true;
    }
    if (ok && !s_abort && pv_pending) issue_pv(ntile - 1);
    if (s_abort) {
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;           // MMA row = entry * 16 + head
    const int e = r >> 4, h = r & 15;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool issuer = (warp == 2 && lane == 0);
    const float LN2 = 0.69314718055994531f;
    // the previous tile's row state, consumed by its deferred epilogue
    int pv_t = 0, pv_slot = 0, pv_g = 0, pv_n = 0;
    bool pv_valid = false;
    float pv_m = 0.f, pv_l = 1.f;

    // store tile j's O / l (bf16) through the staging tile with TMA, and its lse
    auto epilogue = [&](int j) -> bool {
      const int ob = j & 1;
      if (!mbar_wait_group(&o_full[ob], (j >> 1) & 1, &s_abort, 2, 128)) return false;
      tc_fence_after();
      if (issuer) bulk_wait_read_all();          // the staging tile has been read by earlier stores
      named_bar_sync(1, 128);
      const float inv = 1.f / pv_l;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float v[32];
        tmem_ld32(lane_addr + 256 + ob * 128 + c4 * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const int col = c4 * 32 + q8 * 8;      // output dims col .. col+7
          uint4 w;
          w.x = pack_bf16(v[q8 * 8 + 0] * inv, v[q8 * 8 + 1] * inv);
          w.y = pack_bf16(v[q8 * 8 + 2] * inv, v[q8 * 8 + 3] * inv);
          w.z = pack_bf16(v[q8 * 8 + 4] * inv, v[q8 * 8 + 5] * inv);
          w.w = pack_bf16(v[q8 * 8 + 6] * inv, v[q8 * 8 + 7] * inv);
          *reinterpret_cast<uint4*>(o_s + (col >> 6) * 16384 + sw128_offset(r, (col & 63) * 2)) = w;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[ob]);
      if (pv_valid)
        a.part_lse[(static_cast<long>(pv_t) * a.Hq + pv_g * ATTP_G + h) * a.topk + pv_slot] =
            (pv_m + log2f(pv_l)) * LN2;
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (issuer) {
        for (int ee = 0; ee < pv_n; ++ee) {
          const int ent = s_ent[j % 3][ee];
          const int y = ((ent >> 6) * a.topk + (ent & 63)) * a.Hq + pv_g * ATTP_G;
          tma_store_2d(&tmap_po, o_s + ee * 2048, 0, y);
          tma_store_2d(&tmap_po, o_s + 16384 + ee * 2048, 64, y);
        }
        bulk_commit();
      }
      return true;
    };

    bool ok = true;
    for (int i = 0; i < ntile && ok; ++i) {   // every exit decision is uniform over the group
      TileInfo ti;
      tile_info(a, tile0 + i, ti);
      const int sb = i & 1;
      const bool valid = e < ti.n;
      int t = 0, slot = 0, p = 0;
      if (valid) {
        const int ent = __ldg(a.entries + ti.e0 + e);
        t = ent >> 6;
        slot = ent & 63;
        const int qs = __ldg(a.q_start + ti.seq), nq = __ldg(a.q_start + ti.seq + 1) - qs;
        p = __ldg(a.ctx_len + ti.seq) - nq + (t - qs);
        if (h == 0) s_ent[i % 3][e] = ent;
      }
      const int vis = valid ? min(128, p - ti.b * a.block_size + 1) : 128;
      // ---- softmax of tile i: scale, mask keys after the query, exp2, row sum
      if (!mbar_wait_group(&s_full[sb], (i >> 1) & 1, &s_abort, 2, 128)) { ok = false; break; }
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float tmp[32];
        tmem_ld32(lane_addr + sb * 128 + c4 * 32, tmp);
#pragma unroll
        for (int c = 0; c < 32; ++c) sv[c4 * 32 + c] = tmp[c];
      }
      tmem_ld_wait();
      float m = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        sv[c] = (c < vis) ? sv[c] * a.scale_log2 : -INFINITY;
        m = fmaxf(m, sv[c]);
      }
      if (!(m > -INFINITY)) m = 0.f;             // only rows past the tile's entries
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);  // S[sb] has been read
      if (!mbar_wait_group(&p_empty[sb], ((i >> 1) & 1) ^ 1, &s_abort, 2, 128)) { ok = false; break; }
      float l = 0.f;
      uint8_t* pbuf = p_s + sb * 32768;
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        float pe[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) { pe[u] = exp2f(sv[c8 * 8 + u] - m); l += pe[u]; }
        uint4 w;
        w.x = pack_bf16(pe[0], pe[1]);
        w.y = pack_bf16(pe[2], pe[3]);
        w.z = pack_bf16(pe[4], pe[5]);
        w.w = pack_bf16(pe[6], pe[7]);
        *reinterpret_cast<uint4*>(pbuf + (c8 >> 3) * 16384 + sw128_offset(r, (c8 & 7) * 16)) = w;
      }
      fence_proxy_async_smem();                  // P visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
      // ---- deferred epilogue of tile i-1 (its PV overlapped this softmax)
      if (i > 0 && !epilogue(i - 1)) { ok = false; break; }
      pv_t = t; pv_slot = slot; pv_g = ti.g; pv_n = ti.n; pv_valid = valid; pv_m = m; pv_l = l;
    }
    if (ok && ntile > 0) epilogue(ntile - 1);
    if (issuer) bulk_wait_all();                 // partial stores complete before exit
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ phase 2
struct MergeArgs {
  const __nv_bfloat16* part_o;   // [total_q][topk][Hq][128]
  const float* part_lse;         // [total_q][Hq][topk]
  const int32_t* block_idx;      // [total_q][Hkv][topk]
  __nv_bfloat16* out;            // [total_q][Hq][128]
  float* lse;                    // [total_q][Hq] or null
  int total_q, Hq, Hkv, topk;
};

// one CTA per (row, group): 16 heads x 16 threads x 8 output dims
__global__ void __launch_bounds__(256) attn_merge_kernel(const MergeArgs a) {
  const int t = blockIdx.x / a.Hkv, g = blockIdx.x % a.Hkv;
  const int h = threadIdx.x >> 4, d8 = threadIdx.x & 15;
  const int head = g * ATTP_G + h;
  const int32_t* sel = a.block_idx + (static_cast<long>(t) * a.Hkv + g) * a.topk;
  const float* pl = a.part_lse + (static_cast<long>(t) * a.Hq + head) * a.topk;
  float mx = -INFINITY;
  for (int s = 0; s < a.topk; ++s)
    if (__ldg(sel + s) >= 0) mx = fmaxf(mx, __ldg(pl + s));
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (mx > -INFINITY) {
    for (int s = 0; s < a.topk; ++s) {
      if (__ldg(sel + s) < 0) continue;
      const float w = __expf(__ldg(pl + s) - mx);
      wsum += w;
      const uint4 o = __ldg(reinterpret_cast<const uint4*>(
          a.part_o + ((static_cast<long>(t) * a.topk + s) * a.Hq + head) * 128 + d8 * 8));
      acc[0] = fmaf(w, bf16lo(o.x), acc[0]); acc[1] = fmaf(w, bf16hi(o.x), acc[1]);
      acc[2] = fmaf(w, bf16lo(o.y), acc[2]); acc[3] = fmaf(w, bf16hi(o.y), acc[3]);
      acc[4] = fmaf(w, bf16lo(o.z), acc[4]); acc[5] = fmaf(w, bf16hi(o.z), acc[5]);
      acc[6] = fmaf(w, bf16lo(o.w), acc[6]); acc[7] = fmaf(w, bf16hi(o.w), acc[7]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4 r;
  r.x = pack_bf16(acc[0] * inv, acc[1] * inv);
  r.y = pack_bf16(acc[2] * inv, acc[3] * inv);
  r.z = pack_bf16(acc[4] * inv, acc[5] * inv);
  r.w = pack_bf16(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(a.out + (static_cast<long>(t) * a.Hq + head) * 128 + d8 * 8) = r;
  if (a.lse && d8 == 0) a.lse[static_cast<long>(t) * a.Hq + head] = wsum > 0.f ? mx + __logf(wsum) : -INFINITY;
}

}  // namespace msa
