// msa_attn_decode: sparse GQA attention for a few queries per sequence over a
// paged KV cache, on the 5th-generation tensor cores.
//
// For query row t (position p, sequence s) and KV group g, query head h of
// the group reads the keys j <= p of the selected blocks (block_idx[t][g][:],
// -1 = empty) from KV head g:  out = softmax(scale * q_h K^T) V,
// lse = log-sum-exp of the scaled logits.  Plain softmax, no sink, no output
// gate (inteligile "MiniMax-M3" model page, rows "Grouped-query attention",
// "Learnable attention sink", "Gated attention output"); the selected-block
// restriction is the "Indexer-selected sparse attention" row; the kernel is the
// decode counterpart daily.dev "Serving options" names ("decode kernels for
// sparse GQA").
//
// A work item is (row, group, split): a split owns a run of at most 8 of the
// row's selected slots.  A decode row has only the 16 query heads of a group,
// too few rows for an MMA, so both products are taken transposed ("swap AB"):
//   S^T = K_b Q^T   (M = 128 keys,  N = 16 heads, K = 128 dims)
//   O^T = V_b^T P^T (M = 128 dims,  N = 16 heads, K = 128 keys)
// with K_b and V_b straight from their TMA tiles (V_b read MN-major, no
// transpose), Q^T and P^T as 16-row K-major tiles, fp32 accumulators in TMEM.
// Each block gets its own max: thread = key reads its 16 head scores from TMEM,
// per-head maxima and sums are warp butterflies plus a 4-warp exchange, and the
// block's O_b^T = V_b^T P_b^T lands in its own TMEM columns.  The item's
// epilogue (thread = output dim) combines its blocks with weights
// exp(m_b - M) ("LSE fusion"); the splits of a row are merged by
// attn_decode_merge_kernel ("Two-phase forward").
//
// Persistent CTAs, one per SM, each walking items blockIdx.x, +gridDim.x, ...:
// warp 0 streams Q and the K/V tiles through a ring of 32 KiB stages (loads
// for the next item start while this one finishes), warp 1 issues the MMAs,
// warps 2-5 run the softmax, warps 6-9 the epilogue of the previous item
// (statistics and O accumulators are double-buffered by item parity).  Every
// wait is bounded.
#pragma once
#include "common.cuh"

namespace msa {

constexpr int ATTD_THREADS = 320;      // warp 0 producer, warp 1 UMMA issuer, warps 2-5 softmax, warps 6-9 epilogue
constexpr int ATTD_G = 16;             // query heads per KV group
constexpr int ATTD_D = 128;            // head_dim
constexpr int ATTD_MAXB = 8;           // selected blocks per work item
constexpr int ATTD_STAGES = 5;         // K / V tiles in flight
constexpr int ATTD_SRING = 8;          // S^T accumulators (TMEM) and P^T tiles (shared memory) in flight
constexpr int ATTD_TILE = 32768;       // one K or V block: [half][128 keys][64 dims] bf16, 128-byte swizzle
constexpr int ATTD_QT = 4096;          // Q (16 heads x 128 dims) or P^T (16 heads x 128 keys), [half][16][64]
constexpr int ATTD_SMEM = ATTD_STAGES * ATTD_TILE + ATTD_SRING * ATTD_QT + 2 * ATTD_QT + 1024;
// TMEM columns: S^T ring at 0 (8 x 16), O_b^T of the item's blocks at 128 + 128 * (item parity) + 16 * b
constexpr uint32_t ATTD_TM_S = 0, ATTD_TM_O = 128;

struct AttnDecodeArgs {
  const int32_t* block_idx;      // [total_q][Hkv][topk]
  __nv_bfloat16* out;            // [total_q][Hq][128]
  float* lse;                    // [total_q][Hq] or null
  const int32_t* q_start;
  const int32_t* ctx_len;
  const int32_t* page_table;
  float* part_o;                 // [units][nsplit][16][128]  (split partials, normalised)
  float* part_lse;               // [units][nsplit][16]       (natural log)
  int4* items;                   // [n_items][6] work-item records (attn_decode_plan_kernel)
  int num_seqs, total_q, Hq, Hkv, topk, max_blocks, num_pages, block_size, nsplit, per, n_items;
  float scale_log2;              // softmax scale * log2(e)
};

// The blocks of one work item, as every role derives them from the same global data.
struct DecItem {
  int t, g, unit, split, n;
  int tile_row[ATTD_MAXB];       // row of K_b / V_b in the [pages * Hkv * 128][128] cache view
  int nvis[ATTD_MAXB];           // visible keys of the block (128 except the query's own block)
};

__device__ __forceinline__ void decode_item(const AttnDecodeArgs& a, int item, DecItem& it, bool report) {
  it.unit = item / a.nsplit;
  it.split = item % a.nsplit;
  it.t = it.unit / a.Hkv;
  it.g = it.unit % a.Hkv;
  const int s = find_seq(a.q_start, a.num_seqs, it.t);
  const int qs = __ldg(a.q_start + s);
  const int nq = __ldg(a.q_start + s + 1) - qs;
  const int p = __ldg(a.ctx_len + s) - nq + (it.t - qs);
  const int slot0 = it.split * a.per, slot1 = min(a.topk, slot0 + a.per);
  it.n = 0;
  for (int slot = slot0; slot < slot1; ++slot) {
    const int b = __ldg(a.block_idx + static_cast<long>(it.unit) * a.topk + slot);
    if (b < 0) continue;
    if (b >= a.max_blocks || b * a.block_size > p) {
      if (report) flag_error(MSA_DEV_BOUNDS);
      continue;
    }
    const int page = __ldg(a.page_table + static_cast<long>(s) * a.max_blocks + b);
    if (page < 0 || page >= a.num_pages) {
      if (report) flag_error(MSA_DEV_BOUNDS);
      continue;
    }
    it.tile_row[it.n] = (page * a.Hkv + it.g) * 128;
    it.nvis[it.n] = min(128, p - b * a.block_size + 1);
    ++it.n;
  }
}

// One thread per work item: its record, so the persistent kernel's roles never walk q_start,
// block_idx and the page table themselves (dependent loads on the issue path).
//   int4 [0] (t, g, unit, split), [1] (n, -, -, -), [2..3] tile_row[0..7], [4..5] nvis[0..7]
__global__ void __launch_bounds__(256) attn_decode_plan_kernel(const AttnDecodeArgs a) {
  const int item = blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= a.n_items) return;
  DecItem it;
  decode_item(a, item, it, true);
  for (int i = it.n; i < ATTD_MAXB; ++i) { it.tile_row[i] = 0; it.nvis[i] = 0; }
  int4* r = a.items + static_cast<long>(item) * 6;
  r[0] = make_int4(it.t, it.g, it.unit, it.split);
  r[1] = make_int4(it.n, 0, 0, 0);
  r[2] = make_int4(it.tile_row[0], it.tile_row[1], it.tile_row[2], it.tile_row[3]);
  r[3] = make_int4(it.tile_row[4], it.tile_row[5], it.tile_row[6], it.tile_row[7]);
  r[4] = make_int4(it.nvis[0], it.nvis[1], it.nvis[2], it.nvis[3]);
  r[5] = make_int4(it.nvis[4], it.nvis[5], it.nvis[6], it.nvis[7]);
}

// A work-item record as loaded by the persistent kernel (six independent 16-byte loads).
struct ItemRec { int4 r[6]; };
__device__ __forceinline__ ItemRec load_item(const AttnDecodeArgs& a, int item) {
  ItemRec x;
  const int4* p = a.items + static_cast<long>(item) * 6;
#pragma unroll
  for (int i = 0; i < 6; ++i) x.r[i] = __ldg(p + i);
  return x;
}
__device__ __forceinline__ int rec_field(const int4& v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// Butterfly reduce-scatter of 16 values over a warp: afterwards lanes 2h and 2h+1 both hold the
// warp's reduction of value h.  16 shuffles instead of 80.
template <bool MAX>
__device__ __forceinline__ float warp_reduce16(const float (&v)[16], int lane) {
  float a8[8], a4[4], a2[2];
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float keep = b4 ? v[8 + j] : v[j], give = b4 ? v[j] : v[8 + j];
    const float o = __shfl_xor_sync(0xFFFFFFFFu, give, 16);
    a8[j] = MAX ? fmaxf(keep, o) : keep + o;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float keep = b3 ? a8[4 + j] : a8[j], give = b3 ? a8[j] : a8[4 + j];
    const float o = __shfl_xor_sync(0xFFFFFFFFu, give, 8);
    a4[j] = MAX ? fmaxf(keep, o) : keep + o;
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float keep = b2 ? a4[2 + j] : a4[j], give = b2 ? a4[j] : a4[2 + j];
    const float o = __shfl_xor_sync(0xFFFFFFFFu, give, 4);
    a2[j] = MAX ? fmaxf(keep, o) : keep + o;
  }
  float r;
  {
    const float keep = b1 ? a2[1] : a2[0], give = b1 ? a2[0] : a2[1];
    const float o = __shfl_xor_sync(0xFFFFFFFFu, give, 2);
    r = MAX ? fmaxf(keep, o) : keep + o;
  }
  const float o = __shfl_xor_sync(0xFFFFFFFFu, r, 1);
  return MAX ? fmaxf(r, o) : r + o;
}

__global__ void __launch_bounds__(ATTD_THREADS, 1)
attn_decode_kernel(const __grid_constant__ CUtensorMap tmap_q,    // q as [total_q*Hq][128]
                   const __grid_constant__ CUtensorMap tmap_k,    // k as [P*Hkv*128][128]
                   const __grid_constant__ CUtensorMap tmap_v,
                   const AttnDecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;                                   // ATTD_STAGES x 32 KiB
  uint8_t* p_s = ring + ATTD_STAGES * ATTD_TILE;          // ATTD_SRING x 4 KiB (P^T tiles)
  uint8_t* q_s = p_s + ATTD_SRING * ATTD_QT;              // 2 x 4 KiB (Q of the item, by item parity)

  __shared__ uint64_t kv_full[ATTD_STAGES], kv_empty[ATTD_STAGES], s_full[ATTD_SRING], s_empty[ATTD_SRING],
      p_full[ATTD_SRING], p_empty[ATTD_SRING], q_full[2], q_empty[2], o_full[2], o_empty[2], st_full[2],
      st_empty[2], drain_bar;
  __shared__ float red_m[2][4][ATTD_G];                   // per-warp block maxima, by block parity
  __shared__ float st_m[2][ATTD_MAXB][ATTD_G];            // per item parity: each block's maxima (scaled, log2)
  __shared__ float st_l[2][ATTD_MAXB][4][ATTD_G];         // and per-warp partial sums of its probabilities
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < ATTD_STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < ATTD_SRING; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 4);
      mbar_init(&st_full[i], 4);
      mbar_init(&st_empty[i], 4);
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
  const int n_local = a.n_items > static_cast<int>(blockIdx.x)
                          ? (a.n_items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer: Q, then K_0 K_1 V_0 K_2 V_1 ... V_n-1
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      const uint64_t pol = l2_policy_evict_first();      // every tile is read once
      uint32_t ring_n = 0;
      int n_q = 0;                                       // Q copies issued
      bool ok = true;
      ItemRec nxt;
      if (n_local > 0) nxt = load_item(a, blockIdx.x);
      for (int li = 0; li < n_local && ok; ++li) {
        const ItemRec it = nxt;                          // the next record loads while this item issues
        if (li + 1 < n_local) nxt = load_item(a, blockIdx.x + (li + 1) * gridDim.x);
        const int it_t = it.r[0].x, it_g = it.r[0].y, it_n = it.r[1].x;
        const int qb = li & 1;
        if (!mbar_wait(&q_empty[qb], ((li >> 1) & 1) ^ 1, &s_abort)) { ok = false; break; }
        mbar_arrive_expect_tx(&q_full[qb], ATTD_QT);
        const int qrow = it_t * a.Hq + it_g * ATTD_G;
        tma_load_2d(q_s + qb * ATTD_QT, &tmap_q, &q_full[qb], 0, qrow);
        tma_load_2d(q_s + qb * ATTD_QT + 2048, &tmap_q, &q_full[qb], 64, qrow);
        ++n_q;
        auto issue = [&](const CUtensorMap* m, int row) -> bool {
          const uint32_t st = ring_n % ATTD_STAGES;
          if (!mbar_wait(&kv_empty[st], ((ring_n / ATTD_STAGES) & 1) ^ 1, &s_abort)) return false;
          mbar_arrive_expect_tx(&kv_full[st], ATTD_TILE);
          tma_load_2d_hint(ring + st * ATTD_TILE, m, &kv_full[st], 0, row, pol);
          tma_load_2d_hint(ring + st * ATTD_TILE + 16384, m, &kv_full[st], 64, row, pol);
          ++ring_n;
          return true;
        };
        for (int i = 0; i <= it_n && ok; ++i) {
          if (i < it_n) ok = issue(&tmap_k, rec_field(it.r[2 + (i >> 2)], i & 3));
          if (ok && i >= 1) ok = issue(&tmap_v, rec_field(it.r[2 + ((i - 1) >> 2)], (i - 1) & 3));
        }
      }
      if (s_abort) {                       // let every issued copy land before the CTA exits
        for (int b = 0; b < 2 && b < n_q; ++b) {
          const int last = b + 2 * ((n_q - 1 - b) / 2);          // last Q copy into buffer b
          mbar_wait_drain(&q_full[b], (last >> 1) & 1);
        }
        for (uint32_t st = 0; st < ATTD_STAGES && st < ring_n; ++st) {
          const uint32_t last = st + ATTD_STAGES * ((ring_n - 1 - st) / ATTD_STAGES);   // last copy into stage st
          mbar_wait_drain(&kv_full[st], (last / ATTD_STAGES) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer: S_0, (S_i, PV_i-1) ..., PV_n-1
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, ATTD_G, false, false);   // A = K_b (K-major), B = Q (K-major)
      const uint32_t id_pv = idesc_bf16(128, ATTD_G, true, false);   // A = V_b^T (MN-major), B = P^T (K-major)
      const uint64_t ring_d = sdesc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t ring_v = sdesc_sw128(smem_u32(ring), 16384, 1024);
      const uint64_t q_d = sdesc_sw128(smem_u32(q_s), 16, 1024);
      const uint64_t p_d = sdesc_sw128(smem_u32(p_s), 16, 1024);
      uint32_t ring_n = 0, sc = 0, pc = 0;
      bool ok = true;
      int n_next = n_local > 0 ? __ldg(&a.items[static_cast<long>(blockIdx.x) * 6 + 1].x) : 0;
      for (int li = 0; li < n_local && ok && !s_abort; ++li) {
        DecItem it;
        it.n = n_next;
        if (li + 1 < n_local) n_next = __ldg(&a.items[static_cast<long>(blockIdx.x + (li + 1) * gridDim.x) * 6 + 1].x);
        const int par = li & 1;
        if (!mbar_wait(&q_full[par], (li >> 1) & 1, &s_abort)) { ok = false; break; }
        tc_fence_after();
        for (int i = 0; i <= it.n && ok; ++i) {
          if (i < it.n) {          // S_i^T = K_i Q^T into the S ring
            const uint32_t st = ring_n % ATTD_STAGES, ss = sc % ATTD_SRING;
            if (!mbar_wait(&kv_full[st], (ring_n / ATTD_STAGES) & 1, &s_abort) ||
                !mbar_wait(&s_empty[ss], ((sc / ATTD_SRING) & 1) ^ 1, &s_abort)) { ok = false; break; }
            tc_fence_after();
            const uint64_t kd = ring_d + ((st * ATTD_TILE) >> 4);
            const uint64_t qd = q_d + ((par * ATTD_QT) >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)   // 16 dims per step; dim halves 16 KiB (K) / 2 KiB (Q) apart
              umma_bf16_ss(tmem + ATTD_TM_S + ss * ATTD_G, kd + (kk >> 2) * 1024 + (kk & 3) * 2,
                           qd + (kk >> 2) * 128 + (kk & 3) * 2, id_s, kk > 0 ? 1u : 0u);
            umma_commit(&s_full[ss]);
            umma_commit(&kv_empty[st]);
            if (i == it.n - 1) umma_commit(&q_empty[par]);
            ++ring_n;
            ++sc;
          }
          if (i >= 1) {            // O_b^T = V_b^T P_b^T into the block's own columns
            const int b = i - 1;
            const uint32_t st = ring_n % ATTD_STAGES, ps = pc % ATTD_SRING;
            if (!mbar_wait(&kv_full[st], (ring_n / ATTD_STAGES) & 1, &s_abort) ||
                !mbar_wait(&p_full[ps], (pc / ATTD_SRING) & 1, &s_abort)) { ok = false; break; }
            if (b == 0 && !mbar_wait(&o_empty[par], ((li >> 1) & 1) ^ 1, &s_abort)) { ok = false; break; }
            tc_fence_after();
            const uint64_t vd = ring_v + ((st * ATTD_TILE) >> 4);
            const uint64_t pd = p_d + ((ps * ATTD_QT) >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: 2 KiB of V rows; key halves of P^T 2 KiB apart
              umma_bf16_ss(tmem + ATTD_TM_O + par * 128 + b * ATTD_G, vd + 128 * kk,
                           pd + (kk >> 2) * 128 + (kk & 3) * 2, id_pv, kk > 0 ? 1u : 0u);
            umma_commit(&kv_empty[st]);
            umma_commit(&p_empty[ps]);
            ++ring_n;
            ++pc;
          }
        }
        if (!ok) break;
        if (it.n == 0) {           // Q arrived but no block of this item is valid
          umma_commit(&q_empty[par]);
          if (!mbar_wait(&o_empty[par], ((li >> 1) & 1) ^ 1, &s_abort)) break;
        }
        umma_commit(&o_full[par]);
      }
      if (s_abort) {
        umma_commit(&drain_bar);
        mbar_wait_drain(&drain_bar, 0);
      }
    }
  } else {
    const int q4 = warp & 3;                             // TMEM lane quarter this warp may access
    const int row = q4 * 32 + lane;                      // key (softmax) / output dim (epilogue)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float c = a.scale_log2;
    const float LN2 = 0.69314718055994531f;
    ItemRec nxt;
    if (n_local > 0) nxt = load_item(a, blockIdx.x);
    if (warp < 6) {
      // ---------------------------------------------------------- softmax: thread = key, one block at a time
      const int sw = warp - 2;                           // 0..3
      const int stid = sw * 32 + lane;
      uint32_t sc = 0;
      for (int li = 0; li < n_local; ++li) {
        const ItemRec x = nxt;
        if (li + 1 < n_local) nxt = load_item(a, blockIdx.x + (li + 1) * gridDim.x);
        const int n = x.r[1].x, par = li & 1;
        // the item's statistics buffer: read by the epilogue of the item two back
        if (!mbar_wait_group(&st_empty[par], ((li >> 1) & 1) ^ 1, &s_abort, 1, 128)) break;
        bool ok = true;
        for (int b = 0; b < n; ++b, ++sc) {
          const uint32_t ss = sc % ATTD_SRING;
          // ---- S_b^T: this key's 16 head scores
          if (!mbar_wait_group(&s_full[ss], (sc / ATTD_SRING) & 1, &s_abort, 1, 128)) { ok = false; break; }
          tc_fence_after();
          float v[16];
          tmem_ld16(lane_addr + ATTD_TM_S + ss * ATTD_G, v);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_empty[ss]);
          const bool vis = row < rec_field(x.r[4 + (b >> 2)], b & 3);   // keys after the query's position do not count
#pragma unroll
          for (int h = 0; h < 16; ++h) v[h] = vis ? v[h] : -INFINITY;
          // ---- per-head maximum over the block's keys
          const float wm = warp_reduce16<true>(v, lane);
          const int rb = b & 1;
          if ((lane & 1) == 0) red_m[rb][sw][lane >> 1] = wm;
          named_bar_sync(1, 128);
          float m[16];
#pragma unroll
          for (int h = 0; h < 16; ++h)
            m[h] = fmaxf(fmaxf(red_m[rb][0][h], red_m[rb][1][h]), fmaxf(red_m[rb][2][h], red_m[rb][3][h])) * c;
          // ---- P^T_b = exp2(c s - max) as bf16 into the P ring ([key half][16 heads][64 keys], swizzled)
          if (!mbar_wait_group(&p_empty[ss], ((sc / ATTD_SRING) & 1) ^ 1, &s_abort, 1, 128)) { ok = false; break; }
          uint8_t* pt = p_s + ss * ATTD_QT + (row >> 6) * 2048;
          float pr[16];
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            pr[h] = exp2f(fmaf(v[h], c, -m[h]));         // exp2(-inf) = 0
            *reinterpret_cast<__nv_bfloat16*>(pt + sw128_offset(h, (row & 63) * 2)) = __float2bfloat16_rn(pr[h]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[ss]);
          const float ws = warp_reduce16<false>(pr, lane);
          if ((lane & 1) == 0) st_l[par][b][sw][lane >> 1] = ws;
          if (stid < 16) st_m[par][b][stid] = m[stid];
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&st_full[par]);       // the item's statistics are written
      }
    } else {
      // ---------------------------------------------------------- epilogue: thread = output dim
      const int etid = (warp - 6) * 32 + lane;           // 0..127
      for (int li = 0; li < n_local; ++li) {
        const ItemRec x = nxt;
        if (li + 1 < n_local) nxt = load_item(a, blockIdx.x + (li + 1) * gridDim.x);
        const int t = x.r[0].x, g = x.r[0].y, unit = x.r[0].z, split = x.r[0].w, n = x.r[1].x, par = li & 1;
        if (!mbar_wait_group(&st_full[par], (li >> 1) & 1, &s_abort, 2, 128) ||
            !mbar_wait_group(&o_full[par], (li >> 1) & 1, &s_abort, 2, 128)) break;
        tc_fence_after();
        float M[16], L[16], acc[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) { M[h] = -INFINITY; L[h] = 0.f; acc[h] = 0.f; }
        for (int b = 0; b < n; ++b)
#pragma unroll
          for (int h = 0; h < 16; ++h) M[h] = fmaxf(M[h], st_m[par][b][h]);
        for (int b = 0; b < n; ++b) {
          float o[16];
          tmem_ld16(lane_addr + ATTD_TM_O + par * 128 + b * ATTD_G, o);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const float w = exp2f(st_m[par][b][h] - M[h]);
            L[h] = fmaf(w, (st_l[par][b][0][h] + st_l[par][b][1][h]) + (st_l[par][b][2][h] + st_l[par][b][3][h]), L[h]);
            acc[h] = fmaf(w, o[h], acc[h]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&o_empty[par]);                    // O columns and statistics free for item li + 2
          mbar_arrive(&st_empty[par]);
        }
        const int head0 = g * ATTD_G;
        if (a.nsplit == 1) {
#pragma unroll
          for (int h = 0; h < 16; ++h)
            a.out[(static_cast<long>(t) * a.Hq + head0 + h) * ATTD_D + row] =
                __float2bfloat16_rn(L[h] > 0.f ? acc[h] / L[h] : 0.f);
          if (a.lse && etid < 16)
            a.lse[static_cast<long>(t) * a.Hq + head0 + etid] = L[etid] > 0.f ? (M[etid] + log2f(L[etid])) * LN2
                                                                               : -INFINITY;
          continue;
        }
        const long pidx = static_cast<long>(unit) * a.nsplit + split;
        float* po = a.part_o + pidx * (ATTD_G * ATTD_D);
#pragma unroll
        for (int h = 0; h < 16; ++h) po[h * ATTD_D + row] = L[h] > 0.f ? acc[h] / L[h] : 0.f;
        if (etid < 16) a.part_lse[pidx * ATTD_G + etid] = L[etid] > 0.f ? (M[etid] + log2f(L[etid])) * LN2 : -INFINITY;
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// The splits of every (row, group), merged by log-sum-exp in split order (deterministic):
// out = sum_s exp(lse_s - L) o_s, L = log sum_s exp(lse_s) ("LSE fusion", "Two-phase forward").
// CTA = (row, group); thread = (head, 8 output dims); every split's values in flight at once.
__global__ void __launch_bounds__(256) attn_decode_merge_kernel(const AttnDecodeArgs a) {
  const int unit = blockIdx.x;
  const int t = unit / a.Hkv, g = unit % a.Hkv;
  const int h = threadIdx.x >> 4, d0 = (threadIdx.x & 15) * 8;
  const float* pl = a.part_lse + static_cast<long>(unit) * a.nsplit * ATTD_G + h;
  const float* po = a.part_o + static_cast<long>(unit) * a.nsplit * (ATTD_G * ATTD_D) + h * ATTD_D + d0;
  float mx = -INFINITY;
  for (int sp = 0; sp < a.nsplit; ++sp) mx = fmaxf(mx, __ldg(pl + sp * ATTD_G));
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (mx > -INFINITY) {
#pragma unroll 4
    for (int sp = 0; sp < a.nsplit; ++sp) {
      const float w = __expf(__ldg(pl + sp * ATTD_G) - mx);
      const float4 o0 = __ldg(reinterpret_cast<const float4*>(po + static_cast<long>(sp) * ATTD_G * ATTD_D));
      const float4 o1 = __ldg(reinterpret_cast<const float4*>(po + static_cast<long>(sp) * ATTD_G * ATTD_D) + 1);
      wsum += w;
      acc[0] = fmaf(w, o0.x, acc[0]); acc[1] = fmaf(w, o0.y, acc[1]); acc[2] = fmaf(w, o0.z, acc[2]); acc[3] = fmaf(w, o0.w, acc[3]);
      acc[4] = fmaf(w, o1.x, acc[4]); acc[5] = fmaf(w, o1.y, acc[5]); acc[6] = fmaf(w, o1.z, acc[6]); acc[7] = fmaf(w, o1.w, acc[7]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4 r;
  r.x = pack_bf16(acc[0] * inv, acc[1] * inv);
  r.y = pack_bf16(acc[2] * inv, acc[3] * inv);
  r.z = pack_bf16(acc[4] * inv, acc[5] * inv);
  r.w = pack_bf16(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(a.out + (static_cast<long>(t) * a.Hq + g * ATTD_G + h) * ATTD_D + d0) = r;
  if (a.lse && (threadIdx.x & 15) == 0)
    a.lse[static_cast<long>(t) * a.Hq + g * ATTD_G + h] = wsum > 0.f ? mx + __logf(wsum) : -INFINITY;
}

}  // namespace msa
