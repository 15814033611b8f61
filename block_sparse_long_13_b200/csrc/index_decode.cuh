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
// page) units.  Warp 0 is the producer: it reads the page ids of 32 units at
// a time (one coalesced load) and streams each unit as H_kv TMA tiles of
// hg x 128 x 64 bf16 (128-byte swizzle) through a ring of shared buffers
// guarded by full/empty mbarriers.  The consumers are groups of 8 warps; a
// group takes every NG-th stage (NG = 2 for at most 2 queries per sequence,
// so one group's per-stage barrier and reduction latency hides behind the
// other's work, 3 for e4m3 keys and one query; else 1).  In a group each
// thread owns one key row, widens it to fp32 and dots it with the
// sequence's (<= 8) queries held in shared
// memory; the block max is a warp redux.sync on order-preserving integer
// keys, then a per-group sum over the heads.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"

namespace msa {

constexpr int IDXD_CONSUMERS = 256;   // threads of one consumer group
// consumer groups for a query bound NQ (the register budget of two groups fits NQ <= 2).  A group's
// time per stage hardly depends on the stage's bytes, so e4m3 keys (half the bytes of a bf16 stage)
// take three groups for one query per sequence.
__host__ __device__ constexpr int idxd_groups(int nq, bool e4m3 = false) {
  return nq <= 1 && e4m3 ? 3 : nq <= 2 ? 2 : 1;
}
__host__ __device__ constexpr int idxd_threads(int nq, bool e4m3 = false) {
  return 32 + IDXD_CONSUMERS * idxd_groups(nq, e4m3);
}
constexpr int IDXD_MAXQ = 8;       // queries per sequence handled by this form
constexpr int IDXD_MAXHG = 8;      // indexer heads per KV group
constexpr int IDXD_MAXHI = 16;     // indexer heads
constexpr int IDXD_MAXSEQ = 2048;  // sequences per call for this form
constexpr int IDXD_SMEM_BUDGET = 212 * 1024;  // dynamic: key ring + each group's queries

struct IdxDecodeArgs {
  const __nv_bfloat16* idx_q;   // [total_q][Hi][64]
  float* scores;                // [total_q][Hkv][max_blocks]
  const int32_t* q_start;
  const int32_t* ctx_len;
  const int32_t* page_table;    // [num_seqs][max_blocks]
  int num_seqs, max_blocks, num_pages, Hi, Hkv, hg, block_size;
  int stage_bytes, stages;
  float k_scale;                // e4m3 keys: value = code * k_scale (1 for bf16 keys)
};

// 16 e4m3 codes (one 16-byte chunk of a key row) widened exactly to fp32: pairs through the
// packed e4m3x2 -> f16x2 conversion, then f16 -> f32 (both exact: every e4m3 value is an f16 value).
__device__ __forceinline__ void e4m3x16_to_f32(const uint4 w, float (&f)[16]) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t lo, hi;
    const uint16_t b01 = static_cast<uint16_t>(words[i] & 0xFFFFu), b23 = static_cast<uint16_t>(words[i] >> 16);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(lo) : "h"(b01));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hi) : "h"(b23));
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    f[4 * i + 0] = a.x; f[4 * i + 1] = a.y; f[4 * i + 2] = b.x; f[4 * i + 3] = b.y;
  }
}

// NQ: compile-time bound on the queries of any sequence (1, 2, 4 or 8).  E4M3: the indexer keys are
// e4m3 codes (64-byte rows, 64-byte TMA swizzle) read back as code * k_scale; else bf16 (128-byte rows,
// 128-byte swizzle).
template <int NQ, bool E4M3 = false>
__global__ void __launch_bounds__(idxd_threads(NQ, E4M3), 1)
index_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, const IdxDecodeArgs a) {
  constexpr int NG = idxd_groups(NQ, E4M3);
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full_bar[16], empty_bar[16];
  __shared__ int s_nbprefix[IDXD_MAXSEQ + 1];
  __shared__ uint32_t s_part[NG][2][NQ][IDXD_MAXHG][4];
  // per consumer group: its current sequence's queries of all heads, fp32, after the key ring
  float* s_q_all = reinterpret_cast<float*>(ring + static_cast<long>(a.stages) * a.stage_bytes);
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

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
    for (int i = 0; i < a.stages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], IDXD_CONSUMERS / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const long total_units = s_nbprefix[a.num_seqs];
  const long u0 = total_units * blockIdx.x / gridDim.x;
  const long u1 = total_units * (blockIdx.x + 1) / gridDim.x;
  const long nstage = (u1 - u0) * a.Hkv;
  if (nstage == 0) return;  // uniform

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

  if (warp == 0) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) tma_prefetch_desc(&tmap_k);
    int page_l = 0;
    uint32_t used = 0, parity_bits = 0;   // per ring slot: issued at least once / parity of the last issue
    // stage k = (unit j, group g) and its ring slot, kept as counters (no 64-bit division per stage)
    long j = 0;
    int g = 0, slot = 0;
    uint32_t par = 0;
    for (long k = 0; k < nstage; ++k) {
      if (k > 0) {
        if (++g == a.Hkv) { g = 0; ++j; }
        if (++slot == a.stages) { slot = 0; par ^= 1u; }
      }
      if (g == 0 && (j & 31) == 0) {      // page ids of the next 32 units, one per lane
        const long uu = u0 + j + lane;
        page_l = 0;
        if (uu < u1) {
          int s, b;
          locate(uu, s, b);
          page_l = __ldg(a.page_table + static_cast<long>(s) * a.max_blocks + b);
          if (page_l < 0 || page_l >= a.num_pages) { flag_error(MSA_DEV_BOUNDS); page_l = 0; }
        }
      }
      const int page = __shfl_sync(0xFFFFFFFFu, page_l, static_cast<int>(j & 31));
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&empty_bar[slot], par ^ 1u, &s_abort);
        if (ok) {
          mbar_arrive_expect_tx(&full_bar[slot], a.stage_bytes);
          tma_load_4d(ring + static_cast<long>(slot) * a.stage_bytes, &tmap_k, &full_bar[slot], 0, 0, g * a.hg,
                      page);
          used |= 1u << slot;
          parity_bits = (parity_bits & ~(1u << slot)) | (par << slot);
        }
      }
      if (__any_sync(0xFFFFFFFFu, !ok)) break;
    }
    if (lane == 0 && s_abort) {  // let issued copies land before the CTA exits
      for (int i = 0; i < a.stages; ++i)
        if (used & (1u << i)) mbar_wait_drain(&full_bar[i], (parity_bits >> i) & 1u);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int c = tid - 32;
    const int grp = c / IDXD_CONSUMERS;   // group: stages k = grp, grp + NG, ...
    const int cl = c % IDXD_CONSUMERS;
    const int cw = cl >> 5;               // warp of the group, 0..7
    const int token = cl & 127;
    const int hl0 = cl >> 7;              // 0 or 1
    const int bar_seq = 1 + 2 * grp, bar_stage = 2 + 2 * grp;   // the group's named barriers
    float* s_q = s_q_all + grp * (NQ * a.Hi * 64);
    int cur_seq = -1, nq = 0, qrow0 = 0, ctx = 0;
    int s, b;
    locate(u0, s, b);
    // the per-group sum of the group's previous stage is made after the barrier that opens the next one
    int pv_nq = 0, pv_row0 = 0, pv_g = 0, pv_b = 0;
    auto combine = [&](int pbuf) {
      if (cl < pv_nq) {
        float tot = 0.f;
        for (int hl = 0; hl < a.hg; ++hl) {
          const uint32_t* pp = s_part[grp][pbuf][cl][hl];
          const float mx = key_to_float(max(max(pp[0], pp[1]), max(pp[2], pp[3])));
          tot += E4M3 ? mx * a.k_scale : mx;    // max_j q . (c_j s) = s max_j q . c_j for s > 0
        }
        a.scores[(static_cast<long>(pv_row0 + cl) * a.Hkv + pv_g) * a.max_blocks + pv_b] = tot;
      }
    };
    bool ok = true;
    int m = 0;                            // stages taken by this group so far
    // stage k = (unit, group g) and its ring slot, kept as counters: a 64-bit division per stage would
    // cost these threads as much as the stage's dot products
    int g = 0, slot = 0;
    uint32_t par = 0;
    auto next_unit = [&]() {              // next block, or next sequence with blocks
      ++b;
      while (b >= s_nbprefix[s + 1] - s_nbprefix[s]) { ++s; b = 0; }
    };
    for (int d = 0; d < grp && grp < nstage; ++d) {   // this group starts at stage grp
      if (++g == a.Hkv) { g = 0; next_unit(); }
      if (++slot == a.stages) { slot = 0; par ^= 1u; }
    }
    for (long k = grp; k < nstage; k += NG, ++m) {
      if (m > 0)
        for (int d = 0; d < NG; ++d) {
          if (++g == a.Hkv) { g = 0; next_unit(); }
          if (++slot == a.stages) { slot = 0; par ^= 1u; }
        }
      if (s != cur_seq) {
        // this sequence's queries (all indexer heads) as fp32
        named_bar_sync(bar_seq, IDXD_CONSUMERS);
        cur_seq = s;
        qrow0 = __ldg(a.q_start + s);
        nq = __ldg(a.q_start + s + 1) - qrow0;
        ctx = __ldg(a.ctx_len + s);
        if (nq > NQ) { if (cl == 0) flag_error(MSA_DEV_BOUNDS); nq = NQ; }
        const int n = nq * a.Hi * 64;
        const __nv_bfloat16* src = a.idx_q + static_cast<long>(qrow0) * a.Hi * 64;
        for (int i = cl; i < n; i += IDXD_CONSUMERS) s_q[i] = __bfloat162float(src[i]);
        named_bar_sync(bar_seq, IDXD_CONSUMERS);
      }
      if (!mbar_wait_group(&full_bar[slot], par, &s_abort, bar_stage, IDXD_CONSUMERS)) { ok = false; break; }
      if (m > 0) combine((m - 1) & 1);
      const uint8_t* tile = ring + static_cast<long>(slot) * a.stage_bytes;
      const int j = b * a.block_size + token;  // absolute key position
      const int pbuf = m & 1;
      for (int hl = hl0; hl < a.hg; hl += 2) {
        float ac0[NQ], ac1[NQ];
#pragma unroll
        for (int i = 0; i < NQ; ++i) { ac0[i] = 0.f; ac1[i] = 0.f; }
        const int h = g * a.hg + hl;
        auto dot8 = [&](const float (&kf)[8], int c0) {      // keys c0 .. c0+7 of the row against the queries
#pragma unroll
          for (int i = 0; i < NQ; ++i) {
            if (NQ == 1 || i < nq) {
              const float4* qp = reinterpret_cast<const float4*>(s_q + (i * a.Hi + h) * 64 + c0);
              const float4 q0 = qp[0], q1 = qp[1];
              float t0 = ac0[i], t1 = ac1[i];
              t0 = fmaf(q0.x, kf[0], t0); t1 = fmaf(q0.y, kf[1], t1); t0 = fmaf(q0.z, kf[2], t0); t1 = fmaf(q0.w, kf[3], t1);
              t0 = fmaf(q1.x, kf[4], t0); t1 = fmaf(q1.y, kf[5], t1); t0 = fmaf(q1.z, kf[6], t0); t1 = fmaf(q1.w, kf[7], t1);
              ac0[i] = t0; ac1[i] = t1;
            }
          }
        };
        if constexpr (E4M3) {
          // this thread's key row: 64 e4m3 codes, 64-byte swizzled (16-byte chunk c of row r at c ^ ((r >> 1) & 3))
          const uint8_t* rowp = tile + (hl * 128 + token) * 64;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((cc ^ ((token >> 1) & 3)) << 4));
            float kf16[16];
            e4m3x16_to_f32(w, kf16);
            const float (&k0)[8] = *reinterpret_cast<const float(*)[8]>(kf16);
            const float (&k1)[8] = *reinterpret_cast<const float(*)[8]>(kf16 + 8);
            dot8(k0, cc * 16);
            dot8(k1, cc * 16 + 8);
          }
        } else {
          // this thread's key row: 64 bf16, 128-byte swizzled
          const uint8_t* rowp = tile + (hl * 128 + token) * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((cc ^ (token & 7)) << 4));
            const float kf[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                                 bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
            dot8(kf, cc * 8);
          }
        }
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
          if (NQ == 1 || i < nq) {
            const int p = ctx - nq + i;
            const float v = (j <= p) ? ac0[i] + ac1[i] : -INFINITY;
            const uint32_t mx = __reduce_max_sync(0xFFFFFFFFu, order_key(v));
            if (lane == 0) s_part[grp][pbuf][i][hl][cw & 3] = mx;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[slot]);  // this warp is done with the tile
      pv_nq = nq; pv_row0 = qrow0; pv_g = g; pv_b = b;
    }
    if (ok && m > 0) {
      named_bar_sync(bar_seq, IDXD_CONSUMERS);          // the group's last partial maxima visible
      combine((m - 1) & 1);
    }
  }
}

}  // namespace msa
