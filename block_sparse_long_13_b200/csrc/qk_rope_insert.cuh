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
// One CTA per row: its r/2 rotation angles are formed once, in double
// precision (positions reach 2^20, where a float product p * theta^(-2i/r)
// would be off by hundredths of a radian), and shared by all the row's heads.
// A warp takes one head at a time: lane l holds channels 4l .. 4l+3 (one 8-byte
// load), the sum of squares is a warp reduction, and the partner of channel
// c < r/2 (channel c + r/2) sits r/8 lanes further on.  Memory-bound: each
// head row is read once and written once.
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
  __shared__ float s_cos[QKR_D / 2], s_sin[QKR_D / 2];
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  __syncthreads();

  // the row's cache slot (checked once; a bad page skips the cache writes, never the queries)
  const int blk = p >= 0 ? p / a.block_size : -1;
  int page = -1;
  if (blk >= 0 && blk < a.max_blocks) page = __ldg(a.page_table + static_cast<long>(s) * a.max_blocks + blk);
  const bool page_ok = page >= 0 && page < a.num_pages;
  if (!page_ok && tid == 0) flag_error(MSA_DEV_BOUNDS);
  const int slot = p >= 0 ? p % a.block_size : 0;

  const int c0 = 4 * lane;                       // this lane's channels c0 .. c0+3
  const int pd = half >> 2;                      // partner distance in lanes (r/8)
  const int partner = lane < pd ? lane + pd : (lane < 2 * pd ? lane - pd : lane);
  for (int j = warp; j < a.Hq + a.Hkv; j += QKR_THREADS / 32) {   // uniform over the warp
    const bool is_q = j < a.Hq;
    const int g = j - a.Hq;
    const __nv_bfloat16* src = is_q ? a.q + (static_cast<long>(t) * a.Hq + j) * QKR_D
                                    : a.k_new + (static_cast<long>(t) * a.Hkv + g) * QKR_D;
    float x[4], w[4];
    load_bf16x4(src + c0, x);
    load_bf16x4((is_q ? a.q_w : a.k_w) + c0, w);
    float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    const float inv = rsqrtf(ss * (1.f / QKR_D) + a.eps);
    float y[4], o4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) y[u] = x[u] * inv * w[u];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float other = __shfl_sync(0xFFFFFFFFu, y[u], partner);   // every lane takes part
      const int c = c0 + u;
      if (c < half) {                            // first of the pair: a cos - b sin
        o4[u] = y[u] * s_cos[c] - other * s_sin[c];
      } else if (c < a.rotary_dim) {             // second of the pair: b cos + a sin
        o4[u] = y[u] * s_cos[c - half] + other * s_sin[c - half];
      } else {
        o4[u] = y[u];
      }
    }
    if (is_q) {
      store_bf16x4(a.q + (static_cast<long>(t) * a.Hq + j) * QKR_D + c0, o4);
    } else if (page_ok) {
      const long row = ((static_cast<long>(page) * a.Hkv + g) * a.block_size + slot) * QKR_D;
      store_bf16x4(a.k_cache + row + c0, o4);
      *reinterpret_cast<uint2*>(a.v_cache + row + c0) =
          *reinterpret_cast<const uint2*>(a.v_new + (static_cast<long>(t) * a.Hkv + g) * QKR_D + c0);
    }
  }
}

}  // namespace msa
