// msa_attn_decode: sparse GQA attention for a few queries per sequence over a
// paged KV cache, split-K over the selected blocks, online-softmax merge.
//
// For query row t (position p, sequence s) and KV group g, query head h of
// the group reads the keys j <= p of the selected blocks (block_idx[t][g][:],
// -1 = empty) from KV head g:  out = softmax(scale * q_h K^T) V,
// lse = log-sum-exp of the scaled logits.  Plain softmax, no sink, no output
// gate (inteligile "MiniMax-M3" model page, rows "Grouped-query attention",
// "Learnable attention sink", "Gated attention output"); the selected-block
// restriction is the "Indexer-selected sparse attention" row.
//
// One CTA per (row, group, split); a split owns a contiguous run of the
// row's selected slots.  Per selected block, one bulk copy brings V_b (32 KiB)
// into shared memory while thread i loads key row i (all 16 pieces in flight)
// and makes its 16 head dot products; for P.V thread (dp, hh) owns output
// dimensions 2dp, 2dp+1 of heads 8hh..8hh+7.  Running max / sum per head
// follow the usual online-softmax recurrence in the log2 domain.  Splits of a unit write
// (O, lse) partials to the workspace; the last split to finish (device
// counter) merges them by log-sum-exp ("LSE fusion", "Two-phase forward").
#pragma once
#include "common.cuh"

namespace msa {

constexpr int ATTD_THREADS = 128;
constexpr int ATTD_G = 16;     // query heads per KV group handled by this kernel
constexpr int ATTD_D = 128;    // head_dim
constexpr int ATTD_VBYTES = 128 * ATTD_D * 2;          // one V block, bf16
constexpr int ATTD_SMEM = ATTD_VBYTES + 128;           // dynamic: V block (+ alignment)

struct AttnDecodeArgs {
  const __nv_bfloat16* q;        // [total_q][Hq][128]
  const __nv_bfloat16* k_cache;  // [P][Hkv][128][128]
  const __nv_bfloat16* v_cache;
  const int32_t* block_idx;      // [total_q][Hkv][topk]
  __nv_bfloat16* out;            // [total_q][Hq][128]
  float* lse;                    // [total_q][Hq] or null
  const int32_t* q_start;
  const int32_t* ctx_len;
  const int32_t* page_table;
  float* part_o;                 // [units][nsplit][16][128]
  float* part_lse;               // [units][nsplit][16]
  int* counters;                 // [units]
  int num_seqs, total_q, Hq, Hkv, topk, max_blocks, num_pages, block_size, nsplit;
  float scale_log2;              // softmax scale * log2(e)
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__global__ void __launch_bounds__(ATTD_THREADS)
attn_decode_kernel(const AttnDecodeArgs a) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __nv_bfloat16* s_v = reinterpret_cast<__nv_bfloat16*>((reinterpret_cast<uintptr_t>(dsm) + 127) & ~uintptr_t(127));
  __shared__ __align__(16) float s_q[ATTD_G * ATTD_D];     // scaled queries (log2 domain)
  __shared__ __align__(16) float s_p[ATTD_G * 128];        // probabilities of the current block
  __shared__ float s_red[4][ATTD_G];
  __shared__ float s_m[ATTD_G], s_l[ATTD_G], s_alpha[ATTD_G];
  __shared__ int s_last;
  __shared__ uint64_t v_full;
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dp = tid & 63, hh = tid >> 6;            // P.V: dims 2dp, 2dp+1 of heads 8hh .. 8hh+7
  const long unit = blockIdx.x / a.nsplit;           // (t, g)
  const int split = blockIdx.x % a.nsplit;
  const int t = static_cast<int>(unit / a.Hkv);
  const int g = static_cast<int>(unit % a.Hkv);
  const int s = find_seq(a.q_start, a.num_seqs, t);
  const int qs = __ldg(a.q_start + s);
  const int nq = __ldg(a.q_start + s + 1) - qs;
  const int p = __ldg(a.ctx_len + s) - nq + (t - qs);

  if (tid == 0) {
    s_abort = 0;
    mbar_init(&v_full, 1);
    fence_mbar_init();
  }
  // queries of the group, pre-scaled into the log2 domain
  const __nv_bfloat16* qg = a.q + (static_cast<long>(t) * a.Hq + g * ATTD_G) * ATTD_D;
  for (int i = tid; i < ATTD_G * ATTD_D; i += ATTD_THREADS) s_q[i] = __bfloat162float(qg[i]) * a.scale_log2;
  if (tid < ATTD_G) { s_m[tid] = -INFINITY; s_l[tid] = 0.f; }
  float o_acc[8][2];
#pragma unroll
  for (int k = 0; k < 8; ++k) { o_acc[k][0] = 0.f; o_acc[k][1] = 0.f; }
  __syncthreads();

  const int per = (a.topk + a.nsplit - 1) / a.nsplit;
  const int slot0 = split * per, slot1 = min(a.topk, slot0 + per);
  const int32_t* sel = a.block_idx + unit * a.topk;
  uint32_t vph = 0;                                  // V copies issued so far (parity of the next wait)
  bool v_pending = false;
  for (int slot = slot0; slot < slot1; ++slot) {
    const int b = __ldg(sel + slot);
    if (b < 0) continue;  // uniform across the CTA
    if (b >= a.max_blocks || b * a.block_size > p) { if (tid == 0) flag_error(MSA_DEV_BOUNDS); continue; }
    int page = __ldg(a.page_table + static_cast<long>(s) * a.max_blocks + b);
    if (page < 0 || page >= a.num_pages) { if (tid == 0) flag_error(MSA_DEV_BOUNDS); continue; }
    const long base = (static_cast<long>(page) * a.Hkv + g) * 128 * ATTD_D;
    // V_b into shared memory (the previous block's readers are past the barrier that ended its loop)
    if (tid == 0) {
      mbar_arrive_expect_tx(&v_full, ATTD_VBYTES);
      bulk_load(s_v, a.v_cache + base, ATTD_VBYTES, &v_full);
    }
    v_pending = true;

    // --- S = q K^T for key tid (16 heads); the row's 16 pieces are loaded before use
    const int j = b * a.block_size + tid;
    const uint4* krow = reinterpret_cast<const uint4*>(a.k_cache + base + static_cast<long>(tid) * ATTD_D);
    uint4 kw[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) kw[c] = __ldg(krow + c);
    float sc[ATTD_G];
#pragma unroll
    for (int h = 0; h < ATTD_G; ++h) sc[h] = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint4 w = kw[c];
      const float kf[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                           bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
      for (int h = 0; h < ATTD_G; ++h) {
        const float4* qp = reinterpret_cast<const float4*>(s_q + h * ATTD_D + c * 8);
        const float4 q0 = qp[0], q1 = qp[1];
        float v = sc[h];
        v = fmaf(q0.x, kf[0], v); v = fmaf(q0.y, kf[1], v); v = fmaf(q0.z, kf[2], v); v = fmaf(q0.w, kf[3], v);
        v = fmaf(q1.x, kf[4], v); v = fmaf(q1.y, kf[5], v); v = fmaf(q1.z, kf[6], v); v = fmaf(q1.w, kf[7], v);
        sc[h] = v;
      }
    }
    const bool vis = j <= p;
    // block max per head
#pragma unroll
    for (int h = 0; h < ATTD_G; ++h) {
      const uint32_t mk = __reduce_max_sync(0xFFFFFFFFu, order_key(vis ? sc[h] : -INFINITY));
      if (lane == 0) s_red[warp][h] = key_to_float(mk);
    }
    __syncthreads();
    if (tid < ATTD_G) {
      const float mb = fmaxf(fmaxf(s_red[0][tid], s_red[1][tid]), fmaxf(s_red[2][tid], s_red[3][tid]));
      const float mo = s_m[tid];
      const float mn = fmaxf(mo, mb);          // finite: the block has >= 1 visible key
      s_alpha[tid] = exp2f(mo - mn);           // 0 on the first block (mo = -inf)
      s_m[tid] = mn;
    }
    __syncthreads();
    // probabilities and their block sums
#pragma unroll
    for (int h = 0; h < ATTD_G; ++h) {
      const float pv = vis ? exp2f(sc[h] - s_m[h]) : 0.f;
      s_p[h * 128 + tid] = pv;
      const float ws = warp_sum(pv);
      if (lane == 0) s_red[warp][h] = ws;
    }
    const bool v_ok = mbar_wait(&v_full, vph & 1, &s_abort);
    ++vph;
    v_pending = !v_ok;
    if (__syncthreads_or(!v_ok)) break;       // s_p, s_red and V_b visible to every thread
    if (tid < ATTD_G) s_l[tid] = s_l[tid] * s_alpha[tid] + (s_red[0][tid] + s_red[1][tid]) + (s_red[2][tid] + s_red[3][tid]);
    // --- O = alpha O + P V, keys in groups of 4 (P as float4), keys past the row's position skipped
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float al = s_alpha[8 * hh + k];
      o_acc[k][0] *= al;
      o_acc[k][1] *= al;
    }
    const uint32_t* vcol = reinterpret_cast<const uint32_t*>(s_v) + dp;   // V[i][2dp .. 2dp+1] at vcol[64 i]
    const float* prow = s_p + (8 * hh) * 128;
    const int nvis = min(128, p - b * a.block_size + 1);
    int i0 = 0;
    for (; i0 + 4 <= nvis; i0 += 4) {
      float4 pw[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) pw[k] = *reinterpret_cast<const float4*>(prow + k * 128 + i0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t vv = vcol[(i0 + u) * 64];
        const float v0 = bf16lo(vv), v1 = bf16hi(vv);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float pk = u == 0 ? pw[k].x : u == 1 ? pw[k].y : u == 2 ? pw[k].z : pw[k].w;
          o_acc[k][0] = fmaf(pk, v0, o_acc[k][0]);
          o_acc[k][1] = fmaf(pk, v1, o_acc[k][1]);
        }
      }
    }
    for (; i0 < nvis; ++i0) {
      const uint32_t vv = vcol[i0 * 64];
      const float v0 = bf16lo(vv), v1 = bf16hi(vv);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float pk = prow[k * 128 + i0];
        o_acc[k][0] = fmaf(pk, v0, o_acc[k][0]);
        o_acc[k][1] = fmaf(pk, v1, o_acc[k][1]);
      }
    }
    __syncthreads();  // s_p / s_l / s_alpha / V_b reused by the next block
  }
  if (s_abort) {                                     // a V copy that did not land in time: let it finish
    if (tid == 0 && v_pending) mbar_wait_drain(&v_full, (vph - 1) & 1);
    return;
  }

  // ---- finish: this split's (O / l, lse)
  const float LN2 = 0.69314718055994531f;
  if (a.nsplit == 1) {
    __nv_bfloat16* orow = a.out + (static_cast<long>(t) * a.Hq + g * ATTD_G) * ATTD_D;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int h = 8 * hh + k;
      const float l = s_l[h];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      *reinterpret_cast<__nv_bfloat162*>(orow + h * ATTD_D + 2 * dp) =
          __floats2bfloat162_rn(o_acc[k][0] * inv, o_acc[k][1] * inv);
    }
    if (a.lse && tid < ATTD_G) {
      const float l = s_l[tid];
      a.lse[static_cast<long>(t) * a.Hq + g * ATTD_G + tid] = l > 0.f ? (s_m[tid] + log2f(l)) * LN2 : -INFINITY;
    }
    return;
  }
  float* po = a.part_o + (unit * a.nsplit + split) * (ATTD_G * ATTD_D);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int h = 8 * hh + k;
    const float l = s_l[h];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    *reinterpret_cast<float2*>(po + h * ATTD_D + 2 * dp) = make_float2(o_acc[k][0] * inv, o_acc[k][1] * inv);
  }
  if (tid < ATTD_G) {
    const float l = s_l[tid];
    a.part_lse[(unit * a.nsplit + split) * ATTD_G + tid] = l > 0.f ? (s_m[tid] + log2f(l)) * LN2 : -INFINITY;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(a.counters + unit, 1) == a.nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge the unit's splits in split order (deterministic)
  if (tid == 0) a.counters[unit] = 0;  // leave the counter ready for the next call
  const volatile float* pl = a.part_lse + unit * a.nsplit * ATTD_G;
  const volatile float* pov = a.part_o + unit * a.nsplit * (ATTD_G * ATTD_D);
  __nv_bfloat16* orow = a.out + (static_cast<long>(t) * a.Hq + g * ATTD_G) * ATTD_D;
  for (int h = 0; h < ATTD_G; ++h) {
    float mx = -INFINITY;
    for (int sp = 0; sp < a.nsplit; ++sp) mx = fmaxf(mx, pl[sp * ATTD_G + h]);
    float wsum = 0.f, acc = 0.f;
    if (mx > -INFINITY) {
      for (int sp = 0; sp < a.nsplit; ++sp) {
        const float w = __expf(pl[sp * ATTD_G + h] - mx);
        wsum += w;
        acc = fmaf(w, pov[(sp * ATTD_G + h) * ATTD_D + tid], acc);
      }
    }
    orow[h * ATTD_D + tid] = __float2bfloat16_rn(wsum > 0.f ? acc / wsum : 0.f);
    if (a.lse && tid == 0)
      a.lse[static_cast<long>(t) * a.Hq + g * ATTD_G + h] = wsum > 0.f ? mx + __logf(wsum) : -INFINITY;
  }
}

}  // namespace msa
