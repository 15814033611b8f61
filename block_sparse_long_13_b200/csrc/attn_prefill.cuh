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
// accumulators in TMEM; two 4-warp softmax groups take alternate tiles, each
// with its own S, P and O in TMEM: thread = row reads its S row, masks keys
// after the query position (only the query's own block has any), writes P as
// bf16 over the first half of its S columns, from where the P V MMA reads it
// (operand A in TMEM: shared-memory bandwidth is left to the S = Q K^T
// operands and the V tile), and later reads its own O accumulator and stores
// O / l (bf16) and lse = m + ln l as the partial of (t, head, slot).  With an
// O per group, one group's epilogue never holds up the other group's P V.
//
// Phase 2 (merge): out(t, h) = sum_slots exp(lse_s - L) O_s with
// L = log sum_s exp(lse_s); lse(t, h) = L.
#pragma once
#include "common.cuh"

namespace msa {

constexpr int ATTP_THREADS = 384;  // warpgroup 0: producer + UMMA warps; warpgroups 1, 2: softmax
// Register split (setmaxnreg): the launch gives 168 per thread (65536 / 384, rounded to 8); warpgroup 0
// returns registers, the softmax warpgroups take them.  128*72 + 256*216 = 64512 = 384*168.
constexpr int ATTP_REGS_CTRL = 72, ATTP_REGS_SOFTMAX = 216;
static_assert(128 * ATTP_REGS_CTRL + 256 * ATTP_REGS_SOFTMAX <= 384 * 168, "register split exceeds the launch");
constexpr int ATTP_TOK = 8;       // tokens per tile (x 16 heads = 128 MMA rows)
constexpr int ATTP_G = 16;        // query heads per KV group
constexpr int ATTP_PHASES = 4;    // tile-list phases walked in lockstep by all CTAs
constexpr int SCHED_ROWS = 32;    // query rows per schedule CTA

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
  int4* tile_rec;             // [max_tiles][4]: one 64-byte record per tile
  const int32_t* page_table;
  int num_seqs, total_q, Hkv, topk, max_blocks, block_size, nbuckets, num_pages, max_tiles;
};

__device__ __forceinline__ int entry_bucket(const SchedArgs& a, int t, int g, int b, int s) {
  return (s * a.Hkv + g) * a.max_blocks + b;
}

// pass = 0: count entries per bucket; pass = 1: scatter them.  Buckets are
// many (sequences x groups x blocks), so the counters are global atomics; the
// order of entries inside a bucket is arbitrary and does not change any result.
// Blocks that most queries select (the planted or sink-like ones, each row's
// own block) would take thousands of atomics on one address, so a CTA first
// gathers its rows' entries per bucket in a shared-memory hash table and then
// adds one count per distinct bucket; each entry's position is the bucket's
// reserved base plus its rank inside the CTA.
constexpr int SCHED_HASH = 4096;                  // table slots: >= 2 x a CTA's entries when it is used
constexpr int SCHED_EPT = SCHED_HASH / 2 / 256;   // entries per thread (256 threads)

__global__ void __launch_bounds__(256) sched_count_scatter_kernel(const SchedArgs a, int pass) {
  __shared__ int s_key[SCHED_HASH];
  __shared__ int s_cnt[SCHED_HASH];               // entries per bucket, then (pass 1) the bucket's base
  const int t0 = blockIdx.x * SCHED_ROWS;
  const int t1 = min(a.total_q, t0 + SCHED_ROWS);
  const int per_row = a.Hkv * a.topk;
  const int nent = (t1 - t0) * per_row;
  const long e0 = static_cast<long>(t0) * per_row;
  // the entry's bucket, or -1 (empty slot or out-of-range index, which is flagged)
  auto bucket_of = [&](int el, int& ent) -> int {
    const int b = __ldg(a.block_idx + e0 + el);
    if (b < 0) return -1;
    const int t = t0 + el / per_row;
    const int rem = el % per_row;
    const int g = rem / a.topk, slot = rem % a.topk;
    const int s = find_seq(a.q_start, a.num_seqs, t);
    const int qs = __ldg(a.q_start + s), nq = __ldg(a.q_start + s + 1) - qs;
    const int p = __ldg(a.ctx_len + s) - nq + (t - qs);
    if (b >= a.max_blocks || b > p / a.block_size) { flag_error(MSA_DEV_BOUNDS); return -1; }
    ent = (t << 6) | slot;
    return entry_bucket(a, t, g, b, s);
  };
  if (2 * SCHED_ROWS * per_row > SCHED_HASH) {    // rows too wide for the table: one atomic per entry
    for (int el = threadIdx.x; el < nent; el += blockDim.x) {
      int ent = 0;
      const int bk = bucket_of(el, ent);
      if (bk < 0) continue;
      if (pass == 0) atomicAdd(&a.counts[bk], 1);
      else a.entries[atomicAdd(&a.cursor[bk], 1)] = ent;
    }
    return;
  }
  for (int i = threadIdx.x; i < SCHED_HASH; i += blockDim.x) { s_key[i] = -1; s_cnt[i] = 0; }
  __syncthreads();
  int hs[SCHED_EPT], li[SCHED_EPT], ents[SCHED_EPT];
#pragma unroll
  for (int k = 0; k < SCHED_EPT; ++k) {
    hs[k] = -1;
    li[k] = 0;
    ents[k] = 0;
    const int el = threadIdx.x + k * 256;
    if (el >= nent) continue;
    const int bk = bucket_of(el, ents[k]);
    if (bk < 0) continue;
    uint32_t h = (static_cast<uint32_t>(bk) * 2654435761u) >> 20;   // 12 bits
    for (int probe = 0; probe < SCHED_HASH; ++probe) {               // the table is at most half full
      const int prev = atomicCAS(&s_key[h], -1, bk);
      if (prev == -1 || prev == bk) { hs[k] = static_cast<int>(h); break; }
      h = (h + 1) & (SCHED_HASH - 1);
    }
    if (hs[k] >= 0) li[k] = atomicAdd(&s_cnt[hs[k]], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < SCHED_HASH; i += blockDim.x) {
    const int bk = s_key[i];
    if (bk < 0) continue;
    if (pass == 0) atomicAdd(&a.counts[bk], s_cnt[i]);
    else s_cnt[i] = atomicAdd(&a.cursor[bk], s_cnt[i]);
  }
  if (pass == 0) return;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < SCHED_EPT; ++k)
    if (hs[k] >= 0) a.entries[s_cnt[hs[k]] + li[k]] = ents[k];
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

// One 64-byte record per tile, so the attention kernel never searches:
//   int[0] bucket, [1] TMA row of K_b / V_b in the cache = (page * Hkv + g) * 128,
//   [2] g, [3] b, [4] position offset of the sequence (p = t + off), [5] entries n,
//   [8 .. 8+n) entries (t << 6 | slot).
__global__ void __launch_bounds__(256) sched_tiles_kernel(const SchedArgs a) {
  const int T = min(a.total_tiles[0], a.max_tiles);
  for (int tile = blockIdx.x * blockDim.x + threadIdx.x; tile < T; tile += gridDim.x * blockDim.x) {
    int lo = 0, hi = a.nbuckets - 1;  // largest bucket with tile_offsets[bucket] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.tile_offsets + mid) <= tile) lo = mid; else hi = mid - 1;
    }
    const int b = lo % a.max_blocks, g = (lo / a.max_blocks) % a.Hkv, seq = lo / (a.max_blocks * a.Hkv);
    const int e0 = __ldg(a.offsets + lo) + (tile - __ldg(a.tile_offsets + lo)) * ATTP_TOK;
    const int n = min(ATTP_TOK, __ldg(a.offsets + lo + 1) - e0);
    int page = __ldg(a.page_table + static_cast<long>(seq) * a.max_blocks + b);
    if (page < 0 || page >= a.num_pages) { flag_error(MSA_DEV_BOUNDS); page = 0; }
    const int off = __ldg(a.ctx_len + seq) - __ldg(a.q_start + seq + 1);
    int ent[ATTP_TOK];
#pragma unroll
    for (int e = 0; e < ATTP_TOK; ++e) ent[e] = e < n ? a.entries[e0 + e] : 0;
    int4* r = a.tile_rec + static_cast<long>(tile) * 4;
    r[0] = make_int4(lo, (page * a.Hkv + g) * 128, g, b);
    r[1] = make_int4(off, n, 0, 0);
    r[2] = make_int4(ent[0], ent[1], ent[2], ent[3]);
    r[3] = make_int4(ent[4], ent[5], ent[6], ent[7]);
  }
}

// ------------------------------------------------------------------ phase 1
struct AttnPrefillArgs {
  const int4* tile_rec;      // [tiles][4] records written by sched_tiles_kernel
  const int* total_tiles;
  float* part_lse;           // [total_q][Hq][topk]
  int Hq, topk, max_tiles;
  float scale_log2;
};

// shared memory plan (bytes, 1024-aligned): Q[3] 96K | K 32K | V 32K | O staging[2] 64K
constexpr int ATTP_QBUF = 3;      // gathered query tiles in flight (the gather latency needs > 2)
constexpr int ATTP_QBYTES = 32768, ATTP_KVBYTES = 32768, ATTP_STAGE = 32768;
constexpr int ATTP_SMEM = ATTP_QBUF * ATTP_QBYTES + 2 * ATTP_KVBYTES + 2 * ATTP_STAGE + 1024;
// TMEM columns: S[w] (fp32) at 0 / 128, P[w] (bf16 pairs) over the first 64 columns of S[w], O[w] (fp32)
// at 256 / 384; w = the softmax warpgroup = the tile's parity
constexpr uint32_t ATTP_TM_S = 0, ATTP_TM_O = 256;

__global__ void __launch_bounds__(ATTP_THREADS, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,     // q as [total_q*Hq][128]
                    const __grid_constant__ CUtensorMap tmap_k,     // k as [P*Hkv*128][128]
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_po,    // partial O as [total_q*topk*Hq][128]
                    const AttnPrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;                                  // 3 x 32 KiB: [half][128 rows][64]
  uint8_t* k_s = q_s + ATTP_QBUF * ATTP_QBYTES;         // [half][128 keys][64]
  uint8_t* v_s = k_s + ATTP_KVBYTES;                    // [half][128 keys][64]
  uint8_t* o_s = v_s + ATTP_KVBYTES;                    // 2 x 32 KiB: [half][128 rows][64 dims]

  // Per warpgroup w (its own tile sequence, so a parity never runs two phases ahead): s_full[w] S is in
  // TMEM, p_full[w] P is in TMEM (one arrival per warp), o_full[w] O[w] holds its tile, o_empty[w] O[w]
  // has been read (one arrival per warp).
  __shared__ uint64_t kv_full, kv_empty, q_full[ATTP_QBUF], q_empty[ATTP_QBUF], s_full[2], p_full[2], o_full[2],
      o_empty[2], drain_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    s_abort = 0;
    mbar_init(&kv_full, 1);
    mbar_init(&kv_empty, 1);
    for (int i = 0; i < ATTP_QBUF; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 4);
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

  // The tile list is cut into ATTP_PHASES equal phases (about one KV group each for a
  // single-sequence prefill); every CTA takes a contiguous share of each phase in turn,
  // so at any time all CTAs gather query rows of the same phase and those rows stay in L2.
  const int T = min(__ldg(a.total_tiles), a.max_tiles);
  static_assert(ATTP_PHASES == 4, "the phase map below is written out for 4 phases");
  auto share = [&](int q, int& start, int& cnt) {
    const long p0 = static_cast<long>(T) * q / ATTP_PHASES, p1 = static_cast<long>(T) * (q + 1) / ATTP_PHASES;
    const long len = p1 - p0;
    start = static_cast<int>(p0 + len * blockIdx.x / gridDim.x);
    cnt = static_cast<int>(len * (blockIdx.x + 1) / gridDim.x - len * blockIdx.x / gridDim.x);
  };
  int s0, n0, s1, n1, s2, n2, s3, n3;
  share(0, s0, n0);
  share(1, s1, n1);
  share(2, s2, n2);
  share(3, s3, n3);
  const int ntile = n0 + n1 + n2 + n3;
  // global tile of this CTA's i-th tile
  auto tile_of = [=](int i) -> int {
    if (i < n0) return s0 + i;
    i -= n0;
    if (i < n1) return s1 + i;
    i -= n1;
    if (i < n2) return s2 + i;
    return s3 + (i - n2);
  };

  if (warp < 4) {
  regs_dec<ATTP_REGS_CTRL>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer warp
    // Tile records arrive 32 at a time (one per lane, a single coalesced load), so no record
    // fetch sits on the issue path; lanes 0..15 issue the tile's query-row copies in parallel.
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
    }
    int cur_bucket = -1;
    uint32_t kvit = 0;
    int kv_parity = -1;
    uint32_t q_used = 0, q_parity_bits = 0;   // lane 0: per query buffer, issued at least once / parity of the last issue
    // A group's query rows are gathered again by every block they selected: keep them in L2; a K/V
    // block is read by the one or two CTAs that walk its bucket: let it go first.
    const uint64_t pol_q = l2_policy_evict_last(), pol_kv = l2_policy_evict_first();
    int4 ra = make_int4(-1, 0, 0, 0), rb = make_int4(0, 0, 0, 0), rc = rb, rd = rb;   // record of tile (batch + lane)
    for (int i = 0; i < ntile; ++i) {
      if (__any_sync(0xFFFFFFFFu, s_abort != 0)) break;
      if ((i & 31) == 0 && i + lane < ntile) {
        const int4* p = a.tile_rec + static_cast<long>(tile_of(i + lane)) * 4;
        ra = __ldg(p); rb = __ldg(p + 1); rc = __ldg(p + 2); rd = __ldg(p + 3);
      }
      const int src = i & 31;
      const int bucket = __shfl_sync(0xFFFFFFFFu, ra.x, src);
      const int kv_y = __shfl_sync(0xFFFFFFFFu, ra.y, src);
      const int g = __shfl_sync(0xFFFFFFFFu, ra.z, src);
      const int n = __shfl_sync(0xFFFFFFFFu, rb.y, src);
      // the tile's entries (t << 6 | slot)
      const int e0 = __shfl_sync(0xFFFFFFFFu, rc.x, src), e1 = __shfl_sync(0xFFFFFFFFu, rc.y, src);
      const int e2 = __shfl_sync(0xFFFFFFFFu, rc.z, src), e3 = __shfl_sync(0xFFFFFFFFu, rc.w, src);
      const int e4 = __shfl_sync(0xFFFFFFFFu, rd.x, src), e5 = __shfl_sync(0xFFFFFFFFu, rd.y, src);
      const int e6 = __shfl_sync(0xFFFFFFFFu, rd.z, src), e7 = __shfl_sync(0xFFFFFFFFu, rd.w, src);
      // next tile's bucket (when its record is in this batch) for the K/V L2 prefetch
      const int nb_bucket = __shfl_sync(0xFFFFFFFFu, ra.x, (src + 1) & 31);
      const int nb_kv_y = __shfl_sync(0xFFFFFFFFu, ra.y, (src + 1) & 31);
      bool ok = true;
      if (bucket != cur_bucket) {
        if (lane == 0) {
          ok = mbar_wait(&kv_empty, (kvit & 1) ^ 1, &s_abort);
          if (ok) {
            mbar_arrive_expect_tx(&kv_full, 2 * ATTP_KVBYTES);
            tma_load_2d_hint(k_s, &tmap_k, &kv_full, 0, kv_y, pol_kv);
            tma_load_2d_hint(k_s + 16384, &tmap_k, &kv_full, 64, kv_y, pol_kv);
            tma_load_2d_hint(v_s, &tmap_v, &kv_full, 0, kv_y, pol_kv);
            tma_load_2d_hint(v_s + 16384, &tmap_v, &kv_full, 64, kv_y, pol_kv);
            kv_parity = kvit & 1;
          }
        }
        ++kvit;
        cur_bucket = bucket;
        if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) break;
      }
      const int qb = i % ATTP_QBUF;
      const uint32_t qpar = static_cast<uint32_t>((i / ATTP_QBUF) & 1);
      if (lane == 0) {
        ok = mbar_wait(&q_empty[qb], qpar ^ 1u, &s_abort);
        if (ok) {
          mbar_arrive_expect_tx(&q_full[qb], n * 4096);
          q_used |= 1u << qb;
          q_parity_bits = (q_parity_bits & ~(1u << qb)) | (qpar << qb);
        }
      }
      if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) break;
      // query rows of the tile's entries (MMA row 16e + head), [half][128 rows][64 dims] swizzled:
      // lane 2e + half issues entry e's half
      {
        const int el = lane >> 1, half = lane & 1;
        const int en = el == 0 ? e0 : el == 1 ? e1 : el == 2 ? e2 : el == 3 ? e3 : el == 4 ? e4 : el == 5 ? e5
                     : el == 6 ? e6 : e7;
        if (lane < 2 * ATTP_TOK && el < n)
          tma_load_2d_hint(q_s + qb * ATTP_QBYTES + half * 16384 + el * 2048, &tmap_q, &q_full[qb], half * 64,
                           (en >> 6) * a.Hq + g * ATTP_G, pol_q);
      }
      // warm L2 with the next bucket's K/V
      if (lane == 0 && i + 1 < ntile && src != 31 && nb_bucket != bucket) {
        tma_prefetch_l2_2d(&tmap_k, 0, nb_kv_y);
        tma_prefetch_l2_2d(&tmap_k, 64, nb_kv_y);
        tma_prefetch_l2_2d(&tmap_v, 0, nb_kv_y);
        tma_prefetch_l2_2d(&tmap_v, 64, nb_kv_y);
      }
    }
    if (lane == 0 && s_abort) {                  // let issued copies land before the CTA exits
      if (kv_parity >= 0) mbar_wait_drain(&kv_full, kv_parity);
      for (int j = 0; j < ATTP_QBUF; ++j)
        if (q_used & (1u << j)) mbar_wait_drain(&q_full[j], (q_parity_bits >> j) & 1u);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ UMMA issuer
    // Tile i: S(i) = Q K^T into S[i % 2] (A and B from shared memory), then O[(i-1) % 2] = P(i-1) V with
    // P(i-1) read from TMEM over the first half of S[(i-1) % 2].  S(i) overwrites the columns P V(i-2)
    // read: this thread issued P V(i-2) first, and its MMAs run in issue order.
    // This one thread's instruction latency is on the critical path: descriptors are built once
    // (only the 14-bit start address, in 16-byte units, moves) and ring positions are counters.
    const uint32_t id_s = idesc_bf16(128, 128, false, false);
    const uint32_t id_pv = idesc_bf16(128, 128, false, true);
    const uint64_t qdesc0 = sdesc_sw128(smem_u32(q_s), 16, 1024);
    const uint64_t kdesc0 = sdesc_sw128(smem_u32(k_s), 16, 1024);
    const uint64_t vdesc0 = sdesc_sw128(smem_u32(v_s), 16384, 1024);
    int qb = 0;
    uint32_t qph = 0;
    int cur_bucket = -1;
    uint32_t kvit = 0;
    bool pv_pending = false;
    auto issue_pv = [&](int j) -> bool {  // O[j%2] = P[j%2] V
      const int pb = j & 1;
      const uint32_t ph = static_cast<uint32_t>((j >> 1) & 1);
      if (!mbar_wait(&p_full[pb], ph, &s_abort)) return false;
      if (!mbar_wait(&o_empty[pb], ph ^ 1u, &s_abort)) return false;   // tile j-2's O has been read
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: 2048 bytes of V rows
        umma_bf16_ts(tmem + ATTP_TM_O + pb * 128, tmem + ATTP_TM_S + pb * 128 + kk * 8, vdesc0 + 128 * kk, id_pv,
                     kk > 0 ? 1u : 0u);
      umma_commit(&o_full[pb]);
      return true;
    };
    bool ok = true;
    int nbucket = ntile > 0 ? __ldg(&a.tile_rec[static_cast<long>(tile_of(0)) * 4].x) : -1;
    for (int i = 0; i < ntile && ok && !s_abort; ++i) {
      const int bucket = nbucket;
      if (i + 1 < ntile) nbucket = __ldg(&a.tile_rec[static_cast<long>(tile_of(i + 1)) * 4].x);
      if (bucket != cur_bucket) {
        if (pv_pending) {  // finish the previous bucket before its K/V is replaced
          if (!issue_pv(i - 1)) break;
          pv_pending = false;
        }
        if (cur_bucket >= 0) umma_commit(&kv_empty);
        if (!mbar_wait(&kv_full, kvit & 1, &s_abort)) break;
        ++kvit;
        cur_bucket = bucket;
      }
      const int sb = i & 1;
      if (!mbar_wait(&q_full[qb], qph, &s_abort)) break;
      tc_fence_after();
      const uint32_t d = tmem + ATTP_TM_S + sb * 128;
      const uint64_t qd = qdesc0 + static_cast<uint64_t>((qb * ATTP_QBYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {   // 16 dims per step: 32 bytes within a 128-byte row, halves 16 KiB apart
        const uint32_t off16 = (kk >> 2) * 1024 + (kk & 3) * 2;
        umma_bf16_ss(d, qd + off16, kdesc0 + off16, id_s, kk > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[sb]);
      umma_commit(&q_empty[qb]);
      if (++qb == ATTP_QBUF) { qb = 0; qph ^= 1u; }
      if (pv_pending) ok = issue_pv(i - 1);
      pv_pending = true;
    }
    if (ok && !s_abort && pv_pending) issue_pv(ntile - 1);
    if (s_abort) {
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  }
  } else {
    regs_inc<ATTP_REGS_SOFTMAX>();
    // ------------------------------------------------------------ two softmax + epilogue warpgroups
    // Warpgroup w takes the CTA's tiles i = w, w + 2, ...; it owns S[w], P[w] and staging buffer w.
    // Every warp runs on its own (its 32 TMEM lanes = 2 entries x 16 heads): it waits, arrives and
    // stores its rows without waiting for the other warps.
    const int w = (warp - 4) >> 2;
    const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;            // MMA row = entry * 16 + head
    const int e = r >> 4, h = r & 15;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float LN2 = 0.69314718055994531f;
    const float sc = a.scale_log2;
    const uint64_t pol_stream = l2_policy_evict_first();
    uint8_t* stage = o_s + w * ATTP_STAGE;
    const int nj = (ntile - w + 1) / 2;
    // the fields this row needs of its tiles, prefetched one tile ahead
    struct RowRec { int g, b, off, n, ent; };
    auto load_row = [&](int tile) -> RowRec {
      const int4* p = a.tile_rec + static_cast<long>(tile) * 4;
      const int4 h0 = __ldg(p);
      const int4 h1 = __ldg(p + 1);
      RowRec rr;
      rr.g = h0.z; rr.b = h0.w; rr.off = h1.x; rr.n = h1.y;
      rr.ent = __ldg(reinterpret_cast<const int*>(p + 2) + e);
      return rr;
    };
    RowRec nxt{};
    if (nj > 0) nxt = load_row(tile_of(w));
    for (int j = 0; j < nj; ++j) {               // exit decisions are uniform over the warp
      const int i = 2 * j + w;
      const RowRec rec = nxt;
      if (j + 1 < nj) nxt = load_row(tile_of(i + 2));
      const bool valid = e < rec.n;
      const int ent = rec.ent;
      const int t = ent >> 6, slot = ent & 63;
      const int vis = valid ? min(128, t + rec.off - rec.b * 128 + 1) : 128;  // visible keys of the block

      // ---- S = Q K^T is in TMEM: the row's 128 scores in registers, max over the visible keys
      if (!mbar_wait_warp(&s_full[w], static_cast<uint32_t>(j & 1), &s_abort)) break;
      tc_fence_after();
      const uint32_t s_addr = lane_addr + ATTP_TM_S + w * 128;
      float v0[32], v1[32], v2[32], v3[32];
      tmem_ld32(s_addr, v0);
      tmem_ld32(s_addr + 32, v1);
      tmem_ld32(s_addr + 64, v2);
      tmem_ld32(s_addr + 96, v3);
      tmem_ld_wait();
      if (vis < 128) {                            // the query's own block: keys after it do not count
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c >= vis) v0[c] = -INFINITY;
          if (32 + c >= vis) v1[c] = -INFINITY;
          if (64 + c >= vis) v2[c] = -INFINITY;
          if (96 + c >= vis) v3[c] = -INFINITY;
        }
      }
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) mx[c & 7] = fmax3(mx[c & 7], fmaxf(v0[c], v1[c]), fmaxf(v2[c], v3[c]));
      const float m = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], fmax3(mx[4], mx[5], mx[6]), mx[7]));
      const float mc = (m > -INFINITY) ? m * sc : 0.f;   // -inf only on rows past the tile's entries
      // ---- P = exp2(scale * S - max) as bf16 pairs into P[w] (TMEM), two halves of 64 keys
      float l0 = 0.f, l1 = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int q2 = 0; q2 < 32; ++q2) {
          const int c = half * 64 + q2 * 2;
          const float x0 = c < 32 ? v0[c] : c < 64 ? v1[c - 32] : c < 96 ? v2[c - 64] : v3[c - 96];
          const float x1 = c + 1 < 32 ? v0[c + 1] : c + 1 < 64 ? v1[c - 31] : c + 1 < 96 ? v2[c - 63] : v3[c - 95];
          const float p0 = exp2f(fmaf(x0, sc, -mc)), p1 = exp2f(fmaf(x1, sc, -mc));   // exp2(-inf) = 0
          if (q2 & 1) l1 += p0 + p1; else l0 += p0 + p1;
          pk[q2] = pack_bf16(p0, p1);
        }
        tmem_st32(lane_addr + ATTP_TM_S + w * 128 + half * 32, pk);   // S columns already in registers
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[w]);
      const float l = l0 + l1;

      // ---- O = P V is in TMEM: read it, release the accumulator, then O / l as bf16 to this warp's rows
      if (!mbar_wait_warp(&o_full[w], static_cast<uint32_t>(j & 1), &s_abort)) break;
      tc_fence_after();
      float o0[32], o1[32], o2[32], o3[32];
      const uint32_t o_addr = lane_addr + ATTP_TM_O + w * 128;
      tmem_ld32(o_addr, o0);
      tmem_ld32(o_addr + 32, o1);
      tmem_ld32(o_addr + 64, o2);
      tmem_ld32(o_addr + 96, o3);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[w]);
      if (lane == 0) bulk_wait_read_all();        // this warp's previous stores have left its staging rows
      __syncwarp();
      const float inv = 1.f / l;
#pragma unroll
      for (int q8 = 0; q8 < 16; ++q8) {
        const int col = q8 * 8;                   // output dims col .. col+7
        const float* ov = q8 < 4 ? o0 + col : q8 < 8 ? o1 + col - 32 : q8 < 12 ? o2 + col - 64 : o3 + col - 96;
        uint4 wv;
        wv.x = pack_bf16(ov[0] * inv, ov[1] * inv);
        wv.y = pack_bf16(ov[2] * inv, ov[3] * inv);
        wv.z = pack_bf16(ov[4] * inv, ov[5] * inv);
        wv.w = pack_bf16(ov[6] * inv, ov[7] * inv);
        *reinterpret_cast<uint4*>(stage + (col >> 6) * 16384 + sw128_offset(r, (col & 63) * 2)) = wv;
      }
      if (valid)
        a.part_lse[(static_cast<long>(t) * a.Hq + rec.g * ATTP_G + h) * a.topk + slot] = (mc + log2f(l)) * LN2;
      fence_proxy_async_smem();
      const int ent_hi = __shfl_sync(0xFFFFFFFFu, ent, 16);   // entry 2*quarter + 1 (lanes 16..31)
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int ee = 2 * quarter + k2;
          if (ee < rec.n) {
            const int en = k2 ? ent_hi : ent;
            const int y = ((en >> 6) * a.topk + (en & 63)) * a.Hq + rec.g * ATTP_G;
            tma_store_2d_hint(&tmap_po, stage + ee * 2048, 0, y, pol_stream);
            tma_store_2d_hint(&tmap_po, stage + 16384 + ee * 2048, 64, y, pol_stream);
          }
        }
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();               // partial stores complete before exit
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

// one CTA per (row, group): 16 heads x 16 threads x 8 output dims.  The 16 threads of a head first read
// the slots' selections and lse values in parallel (thread j: slots j, j + 16, ...), so the CTA pays one
// round trip for them instead of one per slot, and leave each slot's weight in shared memory.
constexpr int MRG_MAXK = 64;   // topk bound of the configuration
__global__ void __launch_bounds__(256) attn_merge_kernel(const MergeArgs a) {
  __shared__ float s_w[ATTP_G][MRG_MAXK];   // per head and slot: exp(lse - max), or -1 (slot not selected)
  const int t = blockIdx.x / a.Hkv, g = blockIdx.x % a.Hkv;
  const int h = threadIdx.x >> 4, d8 = threadIdx.x & 15;
  const int head = g * ATTP_G + h;
  const int32_t* sel = a.block_idx + (static_cast<long>(t) * a.Hkv + g) * a.topk;
  const float* pl = a.part_lse + (static_cast<long>(t) * a.Hq + head) * a.topk;
  float mx = -INFINITY;
  for (int s = d8; s < a.topk; s += 16)
    if (__ldg(sel + s) >= 0) mx = fmaxf(mx, __ldg(pl + s));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));   // the head's 16 lanes
  for (int s = d8; s < a.topk; s += 16)
    s_w[h][s] = __ldg(sel + s) >= 0 ? (mx > -INFINITY ? __expf(__ldg(pl + s) - mx) : 0.f) : -1.f;
  __syncwarp();                             // a head's 16 threads share one warp
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (mx > -INFINITY) {
    // 8 slots per round, every partial load of the round issued before the first is used
    const __nv_bfloat16* po = a.part_o + (static_cast<long>(t) * a.topk * a.Hq + head) * 128 + d8 * 8;
    for (int s0 = 0; s0 < a.topk; s0 += 8) {
      uint4 o[8];
      float w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int s = s0 + k;
        w[k] = s < a.topk ? s_w[h][s] : -1.f;
        o[k] = w[k] >= 0.f ? __ldcs(reinterpret_cast<const uint4*>(po + static_cast<long>(s) * a.Hq * 128))
                           : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (w[k] < 0.f) continue;
        wsum += w[k];
        acc[0] = fmaf(w[k], bf16lo(o[k].x), acc[0]); acc[1] = fmaf(w[k], bf16hi(o[k].x), acc[1]);
        acc[2] = fmaf(w[k], bf16lo(o[k].y), acc[2]); acc[3] = fmaf(w[k], bf16hi(o[k].y), acc[3]);
        acc[4] = fmaf(w[k], bf16lo(o[k].z), acc[4]); acc[5] = fmaf(w[k], bf16hi(o[k].z), acc[5]);
        acc[6] = fmaf(w[k], bf16lo(o[k].w), acc[6]); acc[7] = fmaf(w[k], bf16hi(o[k].w), acc[7]);
      }
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
