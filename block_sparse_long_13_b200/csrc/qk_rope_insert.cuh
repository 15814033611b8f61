// msa_qknorm_rope_insert: the step just before the MSA path, fused.
//
// For every new row t (sequence s, absolute position p):
//   q[t][h]                                <- rope(rmsnorm(q[t][h]) * q_norm_w)      (in place)
//   k_cache[page][g][p % bs]               <- rope(rmsnorm(k_new[t][g]) * k_norm_w)
//   v_cache[page][g][p % bs]               <- v_new[t][g],   page = page_table[s][p / bs]
// rmsnorm: x / sqrt(mean of x^2 over the head's channels + eps) ("MiniMax-M3",
// inteligile model page, row "QK normalization": per-head RMSNorm on queries
// and keys before the rotary embedding); rope: channel pairs (i, i + r/2),
// i < r/2, turn by p * theta^(-2i/r), channels from r = rotary_dim on pass
// through (row "Partial RoPE": partial_rotary_factor 0.5, rotary_dim 64).
// daily.dev "MiniMax M3 ...", section "Serving options", names the fused
// QKNorm + RoPE + KV insert kernel.
//
// One CTA per row.  The row's inputs are contiguous (q: Hq x 256 B, the new k
// and v rows: Hkv x 256 B each), so one thread starts three bulk copies into
// shared memory before anything else, and the row's rotation angles (formed
// once, in double precision: positions reach 2^20, where a float product
// p * theta^(-2i/r) would be off by hundredths of a radian) are computed while
// they fly.  Half a warp takes one head: lane j holds two 4-channel quads of
// it, chosen so that a rotation pair (c, c + r/2) sits in one lane (lanes
// 0 .. r/8-1 hold quads j and j + r/8; the others hold two pass-through
// quads), so the rotation needs no exchange and the sum of squares is a
// 16-lane reduction.  Results are written back in place in shared memory and
// leave by bulk copies: the q row in one, each k and v row of the cache in one.
#pragma once
#include "common.cuh"

namespace msa {

constexpr int QKR_THREADS = 256;
constexpr int QKR_D = 128;     // head_dim

struct QkRopeArgs {
  __nv_bfloat16* q;              // [total_q][Hq][128]    in / out
  const __nv_bfloat16* k_new;    // [total_q][Hkv][128]
  const __nv_bfloat16* v_new;    // [total_q][Hkv][128]
  const __nv_bfloat16* q_w;      // [128]
  const __nv_bfloat16* k_w;      // [128]
  __nv_bfloat16* k_cache;        // [pages][Hkv][bs][128]
  __nv_bfloat16* v_cache;
  const int32_t* q_start;
  const int32_t* ctx_len;
  const int32_t* page_table;     // [num_seqs][max_blocks]
  int num_seqs, total_q, Hq, Hkv, max_blocks, num_pages, block_size, rotary_dim;
  double log2_theta;
  float eps;
};

// dynamic shared memory of one CTA: the row's q, new k and new v heads
__host__ __device__ constexpr int qkr_smem_bytes(int Hq, int Hkv) { return (Hq + 2 * Hkv) * QKR_D * 2; }

__device__ __forceinline__ void load_bf16x4(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
}
__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* p, const float (&x)[4]) {
  uint2 w;
  w.x = pack_bf16(x[0], x[1]);
  w.y = pack_bf16(x[2], x[3]);
  *reinterpret_cast<uint2*>(p) = w;
}

__global__ void __launch_bounds__(QKR_THREADS) qk_rope_insert_kernel(const QkRopeArgs a) {
  extern __shared__ __align__(128) uint8_t qkr_dsmem[];
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(qkr_dsmem);   // [Hq + Hkv][128]: q heads, then k heads
  __nv_bfloat16* vs = xs + (a.Hq + a.Hkv) * QKR_D;                    // [Hkv][128]
  __shared__ float s_cos[QKR_D / 2], s_sin[QKR_D / 2];
  __shared__ __align__(16) float s_w[2 * QKR_D];   // q_norm_w, then k_norm_w
  __shared__ uint64_t s_bar;
  __shared__ volatile int s_abort;
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t q_bytes = static_cast<uint32_t>(a.Hq) * QKR_D * 2, kv_bytes = static_cast<uint32_t>(a.Hkv) * QKR_D * 2;
  __nv_bfloat16* q_row = a.q + static_cast<long>(t) * a.Hq * QKR_D;
  if (tid == 0) {
    s_abort = 0;
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&s_bar, q_bytes + 2 * kv_bytes);
    bulk_load(xs, q_row, q_bytes, &s_bar);
    bulk_load(xs + a.Hq * QKR_D, a.k_new + static_cast<long>(t) * a.Hkv * QKR_D, kv_bytes, &s_bar);
    bulk_load(vs, a.v_new + static_cast<long>(t) * a.Hkv * QKR_D, kv_bytes, &s_bar);
  }
  const int s = find_seq(a.q_start, a.num_seqs, t);
  const int qs = __ldg(a.q_start + s), nq = __ldg(a.q_start + s + 1) - qs;
  const int p = __ldg(a.ctx_len + s) - nq + (t - qs);
  const int half = a.rotary_dim >> 1;
  if (tid < half) {
    // angle of pair i: p * theta^(-2i/r) = p * 2^(-(2i/r) log2 theta), in double
    const double ang = static_cast<double>(p) * exp2(-(2.0 * tid / a.rotary_dim) * a.log2_theta);
    double sn, cs;
    sincos(ang, &sn, &cs);
    s_cos[tid] = static_cast<float>(cs);
    s_sin[tid] = static_cast<float>(sn);
  }

  // the row's cache slot (checked once; a bad page skips the cache writes, never the queries)
  const int blk = p >= 0 ? p / a.block_size : -1;
  int page = -1;
  if (blk >= 0 && blk < a.max_blocks) page = __ldg(a.page_table + static_cast<long>(s) * a.max_blocks + blk);
  const bool page_ok = page >= 0 && page < a.num_pages;
  if (!page_ok && tid == 0) flag_error(MSA_DEV_BOUNDS);
  const int slot = p >= 0 ? p % a.block_size : 0;
  const long kv_row = page_ok ? ((static_cast<long>(page) * a.Hkv) * a.block_size + slot) * QKR_D : 0;
  const long kv_head = static_cast<long>(a.block_size) * QKR_D;   // elements between a page's KV heads

  // this lane's quads: a rotation pair (qa, qa + r/8) or two pass-through quads
  const int hl = lane & 15, P = a.rotary_dim >> 3;
  const bool rot = hl < P;
  const int qa = rot ? hl : 2 * P + 2 * (hl - P);
  const int qb = rot ? hl + P : qa + 1;
  const int ca = 4 * qa, cb = 4 * qb;
  if (tid < 2 * QKR_D) s_w[tid] = __bfloat162float(tid < QKR_D ? a.q_w[tid] : a.k_w[tid - QKR_D]);
  __syncthreads();                               // the barrier's init and the angles are visible
  // one thread waits for the copies (the others sleep in the barrier instead of spinning on it); after
  // a timed-out wait it lets them land before the CTA leaves
  if (tid == 0 && !mbar_wait(&s_bar, 0, &s_abort)) mbar_wait_drain(&s_bar, 0);
  __syncthreads();
  if (s_abort) return;
  if (tid == 0 && page_ok) {                     // v rows go to the cache untouched
    for (int g = 0; g < a.Hkv; ++g) bulk_store(a.v_cache + kv_row + g * kv_head, vs + g * QKR_D, QKR_D * 2);
  }
  float cs[4], sn[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    cs[u] = rot ? s_cos[ca + u] : 1.f;
    sn[u] = rot ? s_sin[ca + u] : 0.f;
  }

  const int nh = a.Hq + a.Hkv;
  for (int j0 = 2 * warp; j0 < nh; j0 += QKR_THREADS / 16) {   // uniform over the warp
    const int j = j0 + (lane >> 4);
    const bool valid = j < nh;
    const bool is_q = j < a.Hq;
    __nv_bfloat16* row = xs + (valid ? j : 0) * QKR_D;
    float xa[4], xb[4];
    load_bf16x4(row + ca, xa);
    load_bf16x4(row + cb, xb);
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) ss += xa[u] * xa[u] + xb[u] * xb[u];
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);   // within the half-warp
    const float inv = rsqrtf(ss * (1.f / QKR_D) + a.eps);
    const float* w = s_w + (is_q ? 0 : QKR_D);
    const float4 w4a = *reinterpret_cast<const float4*>(w + ca), w4b = *reinterpret_cast<const float4*>(w + cb);
    const float wa[4] = {w4a.x, w4a.y, w4a.z, w4a.w}, wb[4] = {w4b.x, w4b.y, w4b.z, w4b.w};
    float oa[4], ob[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float ya = xa[u] * inv * wa[u];
      const float yb = xb[u] * inv * wb[u];
      // first of a pair: a cos - b sin; second: b cos + a sin (pass-through quads: cos 1, sin 0)
      oa[u] = rot ? ya * cs[u] - yb * sn[u] : ya;
      ob[u] = rot ? yb * cs[u] + ya * sn[u] : yb;
    }
    if (valid) {
      store_bf16x4(row + ca, oa);
      store_bf16x4(row + cb, ob);
    }
  }
  fence_proxy_async_smem();                      // the results are read by the bulk copies below
  __syncthreads();
  if (tid == 0) {
    bulk_store(q_row, xs, q_bytes);
    if (page_ok)
      for (int g = 0; g < a.Hkv; ++g)
        bulk_store(a.k_cache + kv_row + g * kv_head, xs + (a.Hq + g) * QKR_D, QKR_D * 2);
    bulk_commit();
    bulk_wait_all();                             // shared memory stays valid until the copies have read it
  }
}

}  // namespace msa
